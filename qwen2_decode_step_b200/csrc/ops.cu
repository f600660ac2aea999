// ops.cu -- the per-operator kernels of the LLAISYS operator list (final
// report, section 3.2, third layer): add, swiglu, embedding, rms_norm (and
// the fused residual-add + RMSNorm), rope, rearrange, and the two-pass
// argmax.  fp32 arithmetic, one rounding to the storage type per output.
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace q2 {

size_t dtype_size(int dtype) { return dtype == Q2_F32 ? 4 : 2; }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// --------------------------------------------------------------------- add
template <typename T>
__global__ void add_kernel(T* c, const T* a, const T* b, size_t n, bool vec) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int V = Storage<T>::kVec;
  size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t nv = vec ? n / V : 0;
  for (size_t i = tid; i < nv; i += stride) {
    float fa[V], fb[V];
    unpack16<T>(reinterpret_cast<const uint4*>(a)[i], fa);
    unpack16<T>(reinterpret_cast<const uint4*>(b)[i], fb);
#pragma unroll
    for (int j = 0; j < V; ++j) fa[j] += fb[j];
    reinterpret_cast<uint4*>(c)[i] = pack16<T>(fa);
  }
  for (size_t i = nv * V + tid; i < n; i += stride) c[i] = from_f<T>(to_f(a[i]) + to_f(b[i]));
}

static dim3 ew_grid(size_t work) {
  size_t blocks = (work + 255) / 256;
  size_t cap = (size_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return dim3((unsigned)blocks);
}

q2_status launch_add(void* c, const void* a, const void* b, size_t n, int dtype, cudaStream_t st) {
  if (n == 0) return Q2_OK;
  bool vec = aligned16(a) && aligned16(b) && aligned16(c);
  if (dtype == Q2_F32)
    Q2_LAUNCH(add_kernel<float>, ew_grid(vec ? n / 4 : n), dim3(256), 0, st, false, (float*)c,
              (const float*)a, (const float*)b, n, vec);
  else
    Q2_LAUNCH(add_kernel<__nv_bfloat16>, ew_grid(vec ? n / 8 : n), dim3(256), 0, st, false,
              (__nv_bfloat16*)c, (const __nv_bfloat16*)a, (const __nv_bfloat16*)b, n, vec);
  return Q2_OK;
}

// ------------------------------------------------------------------ swiglu
// silu(g) * u with the accurate expf (the fast __expf loses ~1e-5 relative at large |g|).
__device__ __forceinline__ float silu_mul(float g, float u) { return u * (g / (1.0f + expf(-g))); }

template <typename T>
__global__ void swiglu_kernel(T* out, const T* gate, const T* up, size_t n, bool vec) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int V = Storage<T>::kVec;
  size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t nv = vec ? n / V : 0;
  for (size_t i = tid; i < nv; i += stride) {
    float g[V], u[V];
    unpack16<T>(reinterpret_cast<const uint4*>(gate)[i], g);
    unpack16<T>(reinterpret_cast<const uint4*>(up)[i], u);
#pragma unroll
    for (int j = 0; j < V; ++j) g[j] = silu_mul(g[j], u[j]);
    reinterpret_cast<uint4*>(out)[i] = pack16<T>(g);
  }
  for (size_t i = nv * V + tid; i < n; i += stride)
    out[i] = from_f<T>(silu_mul(to_f(gate[i]), to_f(up[i])));
}

q2_status launch_swiglu(void* out, const void* gate, const void* up, size_t n, int dtype,
                        cudaStream_t st) {
  if (n == 0) return Q2_OK;
  bool vec = aligned16(out) && aligned16(gate) && aligned16(up);
  if (dtype == Q2_F32)
    Q2_LAUNCH(swiglu_kernel<float>, ew_grid(vec ? n / 4 : n), dim3(256), 0, st, false,
              (float*)out, (const float*)gate, (const float*)up, n, vec);
  else
    Q2_LAUNCH(swiglu_kernel<__nv_bfloat16>, ew_grid(vec ? n / 8 : n), dim3(256), 0, st, false,
              (__nv_bfloat16*)out, (const __nv_bfloat16*)gate, (const __nv_bfloat16*)up, n, vec);
  return Q2_OK;
}

// Rows of interleaved gate/up values (row stride 2I: element 2i is gate i,
// element 2i+1 is up i) -> out [T, I].
template <typename T>
__global__ void swiglu_interleaved_kernel(T* out, const T* gu, int I) {
  pdl_launch_dependents();
  pdl_wait();
  int t = blockIdx.y;
  const T* g = gu + (size_t)t * 2 * I;
  T* o = out + (size_t)t * I;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < I; i += gridDim.x * blockDim.x)
    o[i] = from_f<T>(silu_mul(to_f(g[2 * i]), to_f(g[2 * i + 1])));
}

q2_status launch_swiglu_interleaved(void* out, const void* gu, int T, int I, int dtype,
                                    cudaStream_t st, bool pdl) {
  if (T == 0) return Q2_OK;
  dim3 grid(ceil_div(I, 256) > 64 ? 64 : ceil_div(I, 256), T);
  if (dtype == Q2_F32)
    Q2_LAUNCH(swiglu_interleaved_kernel<float>, grid, dim3(256), 0, st, pdl, (float*)out,
              (const float*)gu, I);
  else
    Q2_LAUNCH(swiglu_interleaved_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, pdl,
              (__nv_bfloat16*)out, (const __nv_bfloat16*)gu, I);
  return Q2_OK;
}

// --------------------------------------------------------------- embedding
// One block per token: a vectorised row copy.  An id outside [0, vocab)
// writes zeros and sets bit 0 of the error flag.
template <typename T>
__global__ void embedding_kernel(T* out, const int64_t* ids, const T* table, long long vocab,
                                 int d, int* err, bool vec) {
  pdl_launch_dependents();
  pdl_wait();
  int t = blockIdx.x;
  long long id = ids[t];
  bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) atomicOr(err, 1);
  T* dst = out + (size_t)t * d;
  const T* src = table + (ok ? (size_t)id * d : 0);
  if (vec) {
    constexpr int V = Storage<T>::kVec;
    for (int i = threadIdx.x; i < d / V; i += blockDim.x)
      reinterpret_cast<uint4*>(dst)[i] = ok ? reinterpret_cast<const uint4*>(src)[i] : make_uint4(0, 0, 0, 0);
  } else {
    for (int i = threadIdx.x; i < d; i += blockDim.x) dst[i] = ok ? src[i] : from_f<T>(0.0f);
  }
}

q2_status launch_embedding(void* out, const int64_t* ids, const void* table, size_t ntok,
                           size_t vocab, size_t d, int dtype, int* err, cudaStream_t st, bool pdl) {
  if (ntok == 0) return Q2_OK;
  size_t es = dtype_size(dtype);
  bool vec = aligned16(out) && aligned16(table) && (d * es) % 16 == 0;
  if (dtype == Q2_F32)
    Q2_LAUNCH(embedding_kernel<float>, dim3((unsigned)ntok), dim3(128), 0, st, pdl, (float*)out,
              ids, (const float*)table, (long long)vocab, (int)d, err, vec);
  else
    Q2_LAUNCH(embedding_kernel<__nv_bfloat16>, dim3((unsigned)ntok), dim3(128), 0, st, pdl,
              (__nv_bfloat16*)out, ids, (const __nv_bfloat16*)table, (long long)vocab, (int)d, err,
              vec);
  return Q2_OK;
}

// ---------------------------------------------------------------- rms_norm
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) s += red[i];
  __syncthreads();
  return s;
}

// One block per row.  residual += y (rounded), then h = w * r / sqrt(mean r^2 + eps).
template <typename T, int NT>
__global__ void __launch_bounds__(NT) add_rms_norm_kernel(T* residual, const T* y, T* h,
                                                          const T* w, int d, float eps) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float red[NT / 32];
  size_t row = blockIdx.x;
  T* r = residual + row * d;
  const T* yr = y ? y + row * d : nullptr;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += NT) {
    float v = to_f(r[i]);
    if (yr) {
      v = round_st<T>(v + to_f(yr[i]));
      r[i] = from_f<T>(v);
    }
    ss += v * v;
  }
  if (!h) return;
  float tot = block_sum<NT>(ss, red);
  float inv = rsqrtf(tot / (float)d + eps);
  T* hr = h + row * d;
  for (int i = threadIdx.x; i < d; i += NT) hr[i] = from_f<T>(to_f(r[i]) * inv * to_f(w[i]));
}

q2_status launch_add_rms_norm(void* residual, const void* y, void* h, const void* w, size_t M,
                              size_t d, float eps, int dtype, cudaStream_t st, bool pdl) {
  if (M == 0) return Q2_OK;
  if (dtype == Q2_F32)
    Q2_LAUNCH(add_rms_norm_kernel<float, 256>, dim3((unsigned)M), dim3(256), 0, st, pdl,
              (float*)residual, (const float*)y, (float*)h, (const float*)w, (int)d, eps);
  else
    Q2_LAUNCH(add_rms_norm_kernel<__nv_bfloat16, 256>, dim3((unsigned)M), dim3(256), 0, st, pdl,
              (__nv_bfloat16*)residual, (const __nv_bfloat16*)y, (__nv_bfloat16*)h,
              (const __nv_bfloat16*)w, (int)d, eps);
  return Q2_OK;
}

template <typename T, int NT>
__global__ void __launch_bounds__(NT) rms_norm_kernel(T* out, const T* in, const T* w, int d,
                                                      float eps) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float red[NT / 32];
  size_t row = blockIdx.x;
  const T* x = in + row * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += NT) {
    float v = to_f(x[i]);
    ss += v * v;
  }
  float tot = block_sum<NT>(ss, red);
  float inv = rsqrtf(tot / (float)d + eps);
  // `out` may alias `in`: every thread reads its own elements before writing them.
  for (int i = threadIdx.x; i < d; i += NT) out[row * d + i] = from_f<T>(to_f(x[i]) * inv * to_f(w[i]));
}

q2_status launch_rms_norm(void* out, const void* in, const void* w, size_t M, size_t d, float eps,
                          int dtype, cudaStream_t st) {
  if (M == 0) return Q2_OK;
  if (dtype == Q2_F32)
    Q2_LAUNCH(rms_norm_kernel<float, 256>, dim3((unsigned)M), dim3(256), 0, st, false,
              (float*)out, (const float*)in, (const float*)w, (int)d, eps);
  else
    Q2_LAUNCH(rms_norm_kernel<__nv_bfloat16, 256>, dim3((unsigned)M), dim3(256), 0, st, false,
              (__nv_bfloat16*)out, (const __nv_bfloat16*)in, (const __nv_bfloat16*)w, (int)d, eps);
  return Q2_OK;
}

// -------------------------------------------------------------------- rope
// One thread per (token, head, pair j).  Angle pos * theta^(-2j/hd) and its
// cosine/sine in double; the rotation itself in fp32.
template <typename T>
__global__ void rope_kernel(T* out, const T* in, const int64_t* pos, long long ntok, int nhead,
                            int hd, double log2_theta) {
  pdl_launch_dependents();
  pdl_wait();
  int half = hd >> 1;
  long long total = ntok * nhead * half;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    int j = (int)(i % half);
    long long th = i / half;  // token * nhead + head
    long long t = th / nhead;
    double ang = (double)pos[t] * exp2(-(2.0 * j / hd) * log2_theta);
    double sd, cd;
    sincos(ang, &sd, &cd);
    float c = (float)cd, s = (float)sd;
    size_t base = (size_t)th * hd;
    float a = to_f(in[base + j]), b = to_f(in[base + j + half]);
    out[base + j] = from_f<T>(a * c - b * s);
    out[base + j + half] = from_f<T>(b * c + a * s);
  }
}

q2_status launch_rope(void* out, const void* in, const int64_t* pos, size_t ntok, size_t nhead,
                      size_t hd, float theta, int dtype, cudaStream_t st) {
  size_t work = ntok * nhead * (hd / 2);
  if (work == 0) return Q2_OK;
  double l2t = log2((double)theta);
  if (dtype == Q2_F32)
    Q2_LAUNCH(rope_kernel<float>, ew_grid(work), dim3(256), 0, st, false, (float*)out,
              (const float*)in, pos, (long long)ntok, (int)nhead, (int)hd, l2t);
  else
    Q2_LAUNCH(rope_kernel<__nv_bfloat16>, ew_grid(work), dim3(256), 0, st, false,
              (__nv_bfloat16*)out, (const __nv_bfloat16*)in, pos, (long long)ntok, (int)nhead,
              (int)hd, l2t);
  return Q2_OK;
}

// --------------------------------------------------------------- rearrange
struct StrideSpec {
  int ndim;
  long long shape[8];
  long long ostr[8];
  long long istr[8];
};

template <int ES>
struct Elem {
  uint8_t b[ES];
};
template <>
struct Elem<16> {
  uint4 v;
};
template <>
struct Elem<8> {
  unsigned long long v;
};
template <>
struct Elem<4> {
  unsigned v;
};
template <>
struct Elem<2> {
  unsigned short v;
};
template <>
struct Elem<1> {
  unsigned char v;
};

template <int ES>
__global__ void rearrange_kernel(void* out, const void* in, StrideSpec s, long long total) {
  using E = Elem<ES>;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    long long rem = i, oo = 0, io = 0;
    for (int d = s.ndim - 1; d >= 0; --d) {
      long long c = rem % s.shape[d];
      rem /= s.shape[d];
      oo += c * s.ostr[d];
      io += c * s.istr[d];
    }
    reinterpret_cast<E*>(out)[oo] = reinterpret_cast<const E*>(in)[io];
  }
}

q2_status launch_rearrange(void* out, const void* in, int ndim, const int64_t* shape,
                           const int64_t* ostr, const int64_t* istr, size_t es, cudaStream_t st) {
  StrideSpec s = {};
  s.ndim = ndim;
  long long total = 1;
  for (int d = 0; d < ndim; ++d) {
    s.shape[d] = shape[d];
    s.ostr[d] = ostr[d];
    s.istr[d] = istr[d];
    total *= shape[d];
  }
  if (total == 0) return Q2_OK;
  // Dense and in the same order on both sides: a plain device-to-device copy
  // (the contiguous fast path the report keeps for the KV write-back).
  bool dense = true;
  long long expect = 1;
  for (int d = ndim - 1; d >= 0; --d) {
    if (shape[d] != 1 && (ostr[d] != expect || istr[d] != expect)) dense = false;
    expect *= shape[d];
  }
  if (dense) {
    Q2_CUDA_TRY(cudaMemcpyAsync(out, in, (size_t)total * es, cudaMemcpyDeviceToDevice, st));
    return Q2_OK;
  }
  dim3 g = ew_grid((size_t)total), b(256);
  switch (es) {
    case 1: Q2_LAUNCH(rearrange_kernel<1>, g, b, 0, st, false, out, in, s, total); break;
    case 2: Q2_LAUNCH(rearrange_kernel<2>, g, b, 0, st, false, out, in, s, total); break;
    case 4: Q2_LAUNCH(rearrange_kernel<4>, g, b, 0, st, false, out, in, s, total); break;
    case 8: Q2_LAUNCH(rearrange_kernel<8>, g, b, 0, st, false, out, in, s, total); break;
    case 16: Q2_LAUNCH(rearrange_kernel<16>, g, b, 0, st, false, out, in, s, total); break;
    default: set_error("rearrange: elem_size must be 1, 2, 4, 8 or 16"); return Q2_ERR_INVALID_ARG;
  }
  return Q2_OK;
}

// ------------------------------------------------------------------ argmax
// Pass 1: block (p, row) scans a slice of the row and writes its best
// (value, index).  Pass 2: one block per row reduces the partials.
template <int NT>
__device__ __forceinline__ void block_argmax(float& v, long long& i, float* rv, long long* ri) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, v, o);
    long long oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (am_better(ov, oi, v, i)) {
      v = ov;
      i = oi;
    }
  }
  int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    rv[w] = v;
    ri[w] = i;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < NT / 32; ++k)
      if (am_better(rv[k], ri[k], v, i)) {
        v = rv[k];
        i = ri[k];
      }
  }
}

template <typename T, int NT>
__global__ void __launch_bounds__(NT) argmax_pass1(const T* x, long long n, int parts,
                                                   float* pv, int64_t* pi) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float rv[NT / 32];
  __shared__ long long ri[NT / 32];
  int p = blockIdx.x;
  size_t row = blockIdx.y;
  long long chunk = (n + parts - 1) / parts;
  long long lo = p * chunk, hi = lo + chunk < n ? lo + chunk : n;
  const T* xr = x + row * n;
  float bv = -INFINITY;
  long long bi = LLONG_MAX;
  for (long long i = lo + threadIdx.x; i < hi; i += NT) {
    float v = to_f(xr[i]);
    if (am_better(v, i, bv, bi)) {
      bv = v;
      bi = i;
    }
  }
  block_argmax<NT>(bv, bi, rv, ri);
  if (threadIdx.x == 0) {
    pv[row * parts + p] = bv;
    pi[row * parts + p] = bi;
  }
}

template <typename T, int NT>
__global__ void __launch_bounds__(NT) argmax_pass2(const float* pv, const int64_t* pi, int parts,
                                                   int64_t* idx, T* val) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float rv[NT / 32];
  __shared__ long long ri[NT / 32];
  size_t row = blockIdx.x;
  float bv = -INFINITY;
  long long bi = LLONG_MAX;
  for (int p = threadIdx.x; p < parts; p += NT) {
    float v = pv[row * parts + p];
    long long i = pi[row * parts + p];
    if (am_better(v, i, bv, bi)) {
      bv = v;
      bi = i;
    }
  }
  block_argmax<NT>(bv, bi, rv, ri);
  if (threadIdx.x == 0) {
    idx[row] = bi;
    if (val) val[row] = from_f<T>(bv);
  }
}

int argmax_parts(size_t rows, size_t n) {
  long long by_size = (long long)((n + 2047) / 2048);
  // enough CTAs to cover the machine several times over (the pass is a
  // latency-bound scan: short per-thread chains matter more than CTA count)
  long long by_sms = (8LL * num_sms() + (long long)rows - 1) / (long long)(rows ? rows : 1);
  long long p = by_size < by_sms ? by_size : by_sms;
  if (p > 256) p = 256;
  if (p < 1) p = 1;
  return (int)p;
}

q2_status launch_argmax(int64_t* idx, void* val, const void* x, size_t rows, size_t n, int dtype,
                        float* pv, int64_t* pi, int parts, cudaStream_t st, bool pdl) {
  if (rows == 0) return Q2_OK;
  dim3 g1(parts, (unsigned)rows);
  if (dtype == Q2_F32) {
    Q2_LAUNCH(argmax_pass1<float, 256>, g1, dim3(256), 0, st, pdl, (const float*)x, (long long)n,
              parts, pv, pi);
    Q2_LAUNCH(argmax_pass2<float, 256>, dim3((unsigned)rows), dim3(256), 0, st, pdl,
              (const float*)pv, (const int64_t*)pi, parts, idx, (float*)val);
  } else {
    Q2_LAUNCH(argmax_pass1<__nv_bfloat16, 256>, g1, dim3(256), 0, st, pdl,
              (const __nv_bfloat16*)x, (long long)n, parts, pv, pi);
    Q2_LAUNCH(argmax_pass2<__nv_bfloat16, 256>, dim3((unsigned)rows), dim3(256), 0, st, pdl,
              (const float*)pv, (const int64_t*)pi, parts, idx, (__nv_bfloat16*)val);
  }
  return Q2_OK;
}

}  // namespace q2
