// api.cu -- the extern "C" operator entry points of q2.h: argument checks,
// then the internal launchers.  Also the thread-local error string and the
// per-device error flag of the operator kernels.
#include <map>
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"
#include "gemm_tc.h"

namespace q2 {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }
void clear_error() { g_last_error.clear(); }

q2_status launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string(what) + ": " + cudaGetErrorString(e));
    return Q2_ERR_CUDA;
  }
  return Q2_OK;
}

// Bit 0: an embedding id outside [0, vocab).  Every device that loads the
// library holds its own copy.
static __device__ int g_op_error;

int* op_error_flag() {
  static std::mutex mu;
  static std::map<int, int*> addr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  auto it = addr.find(dev);
  if (it != addr.end()) return it->second;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_op_error) != cudaSuccess) return nullptr;
  addr[dev] = static_cast<int*>(p);
  return static_cast<int*>(p);
}

// The operator entry's work-split scratch for the tensor-core attention: one
// per device, allocated and its counters zeroed on first use, then kept.  A
// call waits for the previous call's attention (an event) before using it, so
// launches on different streams never share the counters at once.
struct TcWs {
  void* p = nullptr;
  cudaEvent_t done = nullptr;
};
static std::mutex g_tcws_mu;
static std::map<int, TcWs> g_tcws;

q2_status device_error_status(int bits, const char* who) {
  std::string msg = std::string(who) + ": ";
  if (bits & kErrTimeout) {
    msg += "a bounded device-side wait ran out (a pipeline or grid-phase dependency never "
           "arrived); the results of the calls since the last check are undefined";
    if (bits & kErrIndex) msg += "; a kernel also saw a token id outside [0, vocab)";
    set_error(msg);
    return Q2_ERR_TIMEOUT;
  }
  set_error(msg + "a kernel saw a token id outside [0, vocab)");
  return Q2_ERR_INDEX;
}

int num_sms() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  cache[dev] = n;
  return n;
}

static bool dtype_valid(int dt) { return dt == Q2_F32 || dt == Q2_BF16; }

}  // namespace q2

using namespace q2;

#define Q2_DTYPE_CHECK(dt) Q2_CHECK_ARG(dtype_valid(dt), Q2_ERR_DTYPE, "dtype must be Q2_F32 or Q2_BF16")

extern "C" {

const char* q2_last_error(void) { return g_last_error.c_str(); }

const char* q2_version(void) { return "q2 0.1 sm_100a"; }

q2_status q2_check_device_error(void* stream) {
  clear_error();
  int* flag = op_error_flag();
  Q2_CHECK_ARG(flag, Q2_ERR_CUDA, "cannot resolve the device error flag");
  cudaStream_t st = as_stream(stream);
  Q2_CUDA_TRY(cudaStreamSynchronize(st));
  int v = 0;
  Q2_CUDA_TRY(cudaMemcpy(&v, flag, sizeof v, cudaMemcpyDeviceToHost));
  if (v) {
    int zero = 0;
    Q2_CUDA_TRY(cudaMemcpy(flag, &zero, sizeof zero, cudaMemcpyHostToDevice));
    return device_error_status(v, "check_device_error");
  }
  return Q2_OK;
}

q2_status q2_test_attn_plan(size_t rows, size_t pos0, size_t nh, int sms, int* out) {
  clear_error();
  Q2_CHECK_ARG(out && rows > 0 && nh > 0 && sms > 0, Q2_ERR_INVALID_ARG,
               "test_attn_plan: NULL out, or rows, nh or sms of 0");
  Q2_CHECK_ARG(rows < (1u << 30) && pos0 < (1u << 30) && nh < (1u << 16) && sms < (1 << 16),
               Q2_ERR_INVALID_ARG, "test_attn_plan: size too large");
  int n_whole = 0, ts = 0;
  attn_tc_plan((int)rows, (int)pos0, (int)nh, sms, true, &n_whole, &ts);
  const int items = (int)((rows + 127) / 128 * nh);
  out[0] = n_whole;
  out[1] = ts;
  out[2] = n_whole + (items - n_whole) * ts;
  out[3] = items;
  out[4] = attn_tc_slot_capacity(sms);
  out[5] = attn_tc_counter_capacity();
  return Q2_OK;
}

q2_status q2_test_gemm_tile(size_t M, size_t N, int sms, int* bn) {
  clear_error();
  Q2_CHECK_ARG(bn && M > 0 && N > 0 && sms > 0 && M < (1u << 30) && N < (1u << 30), Q2_ERR_INVALID_ARG,
               "test_gemm_tile: NULL bn, sizes of 0 or past 2^30, or no SMs");
  *bn = tc_gemm_token_tile((int)M, (int)N, sms);
  return Q2_OK;
}

q2_status q2_test_raise_device_error(int bits, void* stream) {
  clear_error();
  Q2_CHECK_ARG(bits > 0 && bits <= (kErrIndex | kErrTimeout), Q2_ERR_INVALID_ARG,
               "test_raise_device_error: bits must be 1, 2 or 3");
  int* flag = op_error_flag();
  Q2_CHECK_ARG(flag, Q2_ERR_CUDA, "cannot resolve the device error flag");
  cudaStream_t st = as_stream(stream);
  int cur = 0;
  Q2_CUDA_TRY(cudaMemcpyAsync(&cur, flag, sizeof cur, cudaMemcpyDeviceToHost, st));
  Q2_CUDA_TRY(cudaStreamSynchronize(st));
  cur |= bits;
  Q2_CUDA_TRY(cudaMemcpyAsync(flag, &cur, sizeof cur, cudaMemcpyHostToDevice, st));
  Q2_CUDA_TRY(cudaStreamSynchronize(st));
  return Q2_OK;
}

q2_status q2_add(void* c, const void* a, const void* b, size_t n, int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(n == 0 || (c && a && b), Q2_ERR_INVALID_ARG, "add: NULL pointer");
  return launch_add(c, a, b, n, dtype, as_stream(stream));
}

q2_status q2_swiglu(void* out, const void* gate, const void* up, size_t n, int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(n == 0 || (out && gate && up), Q2_ERR_INVALID_ARG, "swiglu: NULL pointer");
  return launch_swiglu(out, gate, up, n, dtype, as_stream(stream));
}

q2_status q2_embedding(void* out, const int64_t* ids, const void* weight, size_t ntok, size_t vocab,
                       size_t d, int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(ntok == 0 || (out && ids && weight), Q2_ERR_INVALID_ARG, "embedding: NULL pointer");
  Q2_CHECK_ARG(vocab > 0 && d > 0, Q2_ERR_SHAPE, "embedding: vocab and d must be positive");
  Q2_CHECK_ARG(ntok < (1u << 31), Q2_ERR_SHAPE, "embedding: too many tokens");
  int* flag = op_error_flag();
  Q2_CHECK_ARG(flag, Q2_ERR_CUDA, "cannot resolve the device error flag");
  return launch_embedding(out, ids, weight, ntok, vocab, d, dtype, flag, as_stream(stream), false);
}

q2_status q2_linear(void* out, const void* in, const void* weight, const void* bias, size_t M,
                    size_t N, size_t K, int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(M == 0 || N == 0 || (out && in && weight), Q2_ERR_INVALID_ARG, "linear: NULL pointer");
  Q2_CHECK_ARG(K > 0, Q2_ERR_SHAPE, "linear: K must be positive");
  Q2_CHECK_ARG(M < (1u << 31) && N < (1u << 31) && K < (1u << 31), Q2_ERR_SHAPE, "linear: size too large");
  return launch_linear(out, in, weight, bias, (int)M, (int)N, (int)K, dtype, dtype, as_stream(stream), false);
}

q2_status q2_test_tc_gemm(void* out, size_t ldo, int out_dtype, int epilogue, const void* x,
                          const void* w, const void* bias, size_t M, size_t N, size_t K,
                          int allow_split, void* stream) {
  clear_error();
  Q2_CHECK_ARG(out_dtype == Q2_BF16 || out_dtype == Q2_F32, Q2_ERR_DTYPE, "tc gemm: bad out dtype");
  Q2_CHECK_ARG(epilogue >= TC_EPI_PLAIN && epilogue <= TC_EPI_RESID, Q2_ERR_INVALID_ARG,
               "tc gemm: bad epilogue");
  Q2_CHECK_ARG(M == 0 || N == 0 || (out && x && w), Q2_ERR_INVALID_ARG, "tc gemm: NULL pointer");
  Q2_CHECK_ARG(M < (1u << 31) && N < (1u << 31) && K < (1u << 31) && ldo < (1u << 31), Q2_ERR_SHAPE,
               "tc gemm: size too large");
  Q2_CHECK_ARG(K > 0 && K % 8 == 0, Q2_ERR_SHAPE, "tc gemm: K must be a positive multiple of 8");
  cudaStream_t st = as_stream(stream);
  float* ws = nullptr;
  size_t ws_bytes = 0;
  if (allow_split && M && N) {
    ws_bytes = (size_t)M * N * sizeof(float) * 16;
    if (cudaMalloc(&ws, ws_bytes) != cudaSuccess) {
      set_error("tc gemm: no memory for the split-K workspace");
      return Q2_ERR_OOM;
    }
  }
  int* flag = op_error_flag();
  Q2_CHECK_ARG(flag, Q2_ERR_CUDA, "cannot resolve the device error flag");
  q2_status s = tc_gemm(out, (int)ldo, out_dtype, epilogue, x, w, bias, (int)M, (int)N, (int)K, st,
                        flag, ws, ws_bytes);
  if (s == Q2_OK) s = q2_check_device_error(stream);
  if (ws) {
    cudaStreamSynchronize(st);
    cudaFree(ws);
  }
  return s;
}

q2_status q2_rms_norm(void* out, const void* in, const void* weight, size_t M, size_t d, float eps,
                      int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(M == 0 || (out && in && weight), Q2_ERR_INVALID_ARG, "rms_norm: NULL pointer");
  Q2_CHECK_ARG(d > 0 && d < (1u << 31), Q2_ERR_SHAPE, "rms_norm: bad d");
  Q2_CHECK_ARG(M < (1u << 31), Q2_ERR_SHAPE, "rms_norm: too many rows");
  return launch_rms_norm(out, in, weight, M, d, eps, dtype, as_stream(stream));
}

q2_status q2_add_rms_norm(void* residual, const void* y, void* h, const void* weight, size_t M,
                          size_t d, float eps, int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(M == 0 || (residual && h && weight), Q2_ERR_INVALID_ARG, "add_rms_norm: NULL pointer");
  Q2_CHECK_ARG(d > 0 && d < (1u << 31), Q2_ERR_SHAPE, "add_rms_norm: bad d");
  Q2_CHECK_ARG(M < (1u << 31), Q2_ERR_SHAPE, "add_rms_norm: too many rows");
  return launch_add_rms_norm(residual, y, h, weight, M, d, eps, dtype, as_stream(stream), false);
}

q2_status q2_rope(void* out, const void* in, const int64_t* pos, size_t ntok, size_t nhead, size_t hd,
                  float theta, int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  Q2_CHECK_ARG(ntok == 0 || nhead == 0 || (out && in && pos), Q2_ERR_INVALID_ARG, "rope: NULL pointer");
  Q2_CHECK_ARG(hd > 0 && hd % 2 == 0, Q2_ERR_SHAPE, "rope: head dim must be even");
  Q2_CHECK_ARG(theta > 0.f, Q2_ERR_INVALID_ARG, "rope: theta must be positive");
  return launch_rope(out, in, pos, ntok, nhead, hd, theta, dtype, as_stream(stream));
}

q2_status q2_rearrange(void* out, const void* in, int ndim, const int64_t* shape,
                       const int64_t* out_strides, const int64_t* in_strides, size_t elem_size,
                       void* stream) {
  clear_error();
  Q2_CHECK_ARG(ndim >= 0 && ndim <= 8, Q2_ERR_SHAPE, "rearrange: ndim must be 0..8");
  Q2_CHECK_ARG(ndim == 0 || (shape && out_strides && in_strides), Q2_ERR_INVALID_ARG,
               "rearrange: NULL shape/strides");
  for (int d = 0; d < ndim; ++d)
    Q2_CHECK_ARG(shape[d] >= 0, Q2_ERR_SHAPE, "rearrange: negative extent");
  Q2_CHECK_ARG(out && in, Q2_ERR_INVALID_ARG, "rearrange: NULL pointer");
  return launch_rearrange(out, in, ndim, shape, out_strides, in_strides, elem_size, as_stream(stream));
}

q2_status q2_argmax(int64_t* max_idx, void* max_val, const void* vals, size_t rows, size_t n,
                    int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  if (rows == 0) return Q2_OK;
  Q2_CHECK_ARG(max_idx && vals, Q2_ERR_INVALID_ARG, "argmax: NULL pointer");
  Q2_CHECK_ARG(n > 0, Q2_ERR_SHAPE, "argmax: empty rows");
  Q2_CHECK_ARG(rows < (1u << 31), Q2_ERR_SHAPE, "argmax: too many rows");
  cudaStream_t st = as_stream(stream);
  int parts = argmax_parts(rows, n);
  size_t np = rows * (size_t)parts;
  void* scratch = nullptr;
  Q2_CUDA_TRY(cudaMallocAsync(&scratch, np * (sizeof(float) + sizeof(int64_t)) + 16, st));
  int64_t* pi = reinterpret_cast<int64_t*>(scratch);
  float* pv = reinterpret_cast<float*>(pi + np);
  q2_status s = launch_argmax(max_idx, max_val, vals, rows, n, dtype, pv, pi, parts, st, false);
  cudaFreeAsync(scratch, st);
  return s;
}

q2_status q2_self_attention(void* out, const void* q, const void* k, const void* v, size_t seqlen,
                            size_t total_len, size_t nh, size_t nkv, size_t hd, float scale,
                            int dtype, void* stream) {
  clear_error();
  Q2_DTYPE_CHECK(dtype);
  if (seqlen == 0) return Q2_OK;
  Q2_CHECK_ARG(out && q && k && v, Q2_ERR_INVALID_ARG, "self_attention: NULL pointer");
  Q2_CHECK_ARG(seqlen <= total_len, Q2_ERR_SHAPE, "self_attention: seqlen > total_len");
  Q2_CHECK_ARG(nkv > 0 && nh % nkv == 0 && nh / nkv <= 8, Q2_ERR_SHAPE,
               "self_attention: need nh % nkv == 0 and nh / nkv <= 8");
  Q2_CHECK_ARG(hd == 32 || hd == 64 || hd == 128, Q2_ERR_SHAPE, "self_attention: hd must be 32, 64 or 128");
  Q2_CHECK_ARG(total_len < (1u << 30) && nh < 65536, Q2_ERR_SHAPE, "self_attention: size too large");
  AttnRows a = {};
  a.q = q;
  a.q_row_stride = (long long)(nh * hd);
  a.k = k;
  a.v = v;
  a.kv_seq_stride = 0;
  a.kv_tok_stride = (long long)(nkv * hd);
  a.kv_head_stride = (long long)hd;
  a.out = out;
  a.out_row_stride = (long long)(nh * hd);
  a.rows = (int)seqlen;
  a.nh = (int)nh;
  a.nkv = (int)nkv;
  a.hd = (int)hd;
  a.base = (int)(total_len - seqlen + 1);
  a.row_step = 1;
  a.lens = nullptr;
  a.seq_is_row = 0;
  a.fixed_seq = 0;
  a.scale = scale;
  cudaStream_t st = as_stream(stream);
  int nsplit = attn_splits(a.rows, a.nkv, (int)total_len);
  size_t bytes = attn_scratch_bytes(a.rows, a.nh, a.hd, nsplit);
  void* scratch = nullptr;
  if (bytes) Q2_CUDA_TRY(cudaMallocAsync(&scratch, bytes, st));
  q2_status s;
  if (attn_tc_supported(a, dtype)) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_tcws_mu);
    TcWs& w = g_tcws[dev];
    if (e == cudaSuccess && !w.p) {
      e = cudaMalloc(&w.p, attn_tc_ws_bytes());
      if (e == cudaSuccess) e = cudaMemsetAsync(w.p, 0, 4096, st);  // the counters
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&w.done, cudaEventDisableTiming);
      if (e != cudaSuccess && w.p) {
        cudaFree(w.p);
        w.p = nullptr;
      }
    } else if (e == cudaSuccess) {
      e = cudaStreamWaitEvent(st, w.done, 0);
    }
    if (e != cudaSuccess) {
      if (scratch) cudaFreeAsync(scratch, st);
      set_error(std::string("self_attention: ") + cudaGetErrorString(e));
      return Q2_ERR_CUDA;
    }
    s = launch_attention(a, nsplit, scratch, dtype, st, false, nullptr, w.p);
    cudaEventRecord(w.done, st);
  } else {
    s = launch_attention(a, nsplit, scratch, dtype, st, false);
  }
  if (scratch) cudaFreeAsync(scratch, st);
  return s;
}

}  // extern "C"
