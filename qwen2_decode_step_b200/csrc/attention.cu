// attention.cu -- causal GQA self-attention over a KV cache, split over the
// keys ("flash-decode"): each CTA takes one query row, one kv head (all the
// nh/nkv query heads that share it) and one slice of the visible keys,
// stages K/V tiles of 64 positions in shared memory (cp.async, double
// buffered), and keeps an online softmax in fp32 (exp2 with the scale folded
// into q).  A combine pass merges the slices' (max, sum, unnormalised
// output) partials in a fixed order, so results are bit-reproducible.
//
// Definition followed: the attention sketch of the Day-0 adaptation tutorial
// (step 5): scores = q k^T * scale, causal mask, stable softmax, times V; the
// LLAISYS final report (section 3.2) computes attention scores in float.
#include <cstdlib>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace q2 {

namespace {
constexpr int kTK = 64;    // keys per tile
constexpr int kGMax = 8;   // query heads per kv head
constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int HD>
struct AttnSmem {
  static constexpr int kRowBytes = HD * (int)sizeof(T);
  static constexpr int kRowPad = kRowBytes + 16;  // padding: conflict-free row-parallel reads
  static constexpr int kChunks = kRowBytes / 16;
  static constexpr size_t kBytes =
      4 * (size_t)kTK * kRowPad + (size_t)(kGMax * HD + kGMax * kTK + 3 * kGMax) * sizeof(float);
};

__device__ __forceinline__ int visible_keys(const AttnRows& a, int r, int seq) {
  return a.base + a.row_step * r + (a.lens ? a.lens[seq] : 0);
}
}  // namespace

template <typename T, int HD>
__global__ void __launch_bounds__(kThreads) attn_split_kernel(AttnRows a, int nsplit,
                                                              float* part_o, float* part_ml) {
  using SM = AttnSmem<T, HD>;
  constexpr int ROWP = SM::kRowPad, CH = SM::kChunks, EV = 16 / (int)sizeof(T);
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* Ks = smem;
  uint8_t* Vs = Ks + 2 * kTK * ROWP;
  float* qs = reinterpret_cast<float*>(Vs + 2 * kTK * ROWP);
  float* S = qs + kGMax * HD;
  float* ms = S + kGMax * kTK;
  float* ls = ms + kGMax;
  float* al = ls + kGMax;

  pdl_launch_dependents();
  pdl_wait();

  const int split = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = a.nh / a.nkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seq = a.seq_is_row ? r : a.fixed_seq;
  const int L = visible_keys(a, r, seq);
  const int ntiles = L > 0 ? (L + kTK - 1) / kTK : 0;
  const int active = min(nsplit, ntiles);
  const int tps = active > 0 ? (ntiles + active - 1) / active : 0;
  const int t0 = split * tps, t1 = min(t0 + tps, ntiles);
  const bool direct = (nsplit == 1);
  const int dp = tid & 63, hp = tid >> 6;  // PV ownership: dims (2dp, 2dp+1), heads hp, hp+2, ...

  if (t0 >= t1) {
    if (direct) {
      T* orow = reinterpret_cast<T*>(a.out) + (size_t)r * a.out_row_stride + (size_t)g * G * HD;
      for (int i = tid; i < G * HD; i += kThreads) orow[i] = from_f<T>(0.f);
    } else if (tid < G) {
      size_t pidx = ((size_t)r * a.nh + g * G + tid) * nsplit + split;
      part_ml[2 * pidx] = -INFINITY;
      part_ml[2 * pidx + 1] = 0.f;
    }
    return;
  }

  const T* qrow = reinterpret_cast<const T*>(a.q) + (size_t)r * a.q_row_stride + (size_t)g * G * HD;
  const float qscale = a.scale * kLog2e;
  for (int i = tid; i < G * HD; i += kThreads) qs[i] = to_f(qrow[i]) * qscale;
  if (tid < G) {
    ms[tid] = -INFINITY;
    ls[tid] = 0.f;
  }
  const T* kb = reinterpret_cast<const T*>(a.k) + (size_t)seq * a.kv_seq_stride + (size_t)g * a.kv_head_stride;
  const T* vb = reinterpret_cast<const T*>(a.v) + (size_t)seq * a.kv_seq_stride + (size_t)g * a.kv_head_stride;

  auto issue = [&](int t, int buf) {
    const int j0 = t * kTK;
    for (int c = tid; c < kTK * CH; c += kThreads) {
      const int j = c / CH, ch = c % CH;
      const bool valid = j0 + j < L;
      const size_t off = (size_t)(valid ? j0 + j : 0) * a.kv_tok_stride;
      cp_async16(Ks + (size_t)(buf * kTK + j) * ROWP + ch * 16,
                 reinterpret_cast<const uint8_t*>(kb + off) + ch * 16, valid);
      cp_async16(Vs + (size_t)(buf * kTK + j) * ROWP + ch * 16,
                 reinterpret_cast<const uint8_t*>(vb + off) + ch * 16, valid);
    }
  };

  float acc[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.f;

  issue(t0, 0);
  cp_async_commit();
  for (int t = t0; t < t1; ++t) {
    const int buf = (t - t0) & 1;
    if (t + 1 < t1) {
      issue(t + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint8_t* Kt = Ks + (size_t)buf * kTK * ROWP;
    const uint8_t* Vt = Vs + (size_t)buf * kTK * ROWP;
    const int jn = min(kTK, L - t * kTK);

    {  // scores s[h][j] = (q_h . k_j) * scale * log2(e); masked -> -inf
      const int j = tid & 63;
      const uint4* krow = reinterpret_cast<const uint4*>(Kt + (size_t)j * ROWP);
      for (int hh = hp; hh < G; hh += 2) {
        const float* qh = qs + hh * HD;
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          float kf[EV];
          unpack16<T>(krow[c], kf);
#pragma unroll
          for (int e = 0; e < EV; ++e) s = fmaf(qh[c * EV + e], kf[e], s);
        }
        S[hh * kTK + j] = (j < jn) ? s : -INFINITY;
      }
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += kThreads / 32) {  // online softmax update per head
      const float v0 = S[hh * kTK + lane], v1 = S[hh * kTK + lane + 32];
      const float mold = ms[hh];
      const float mnew = fmaxf(mold, warp_max(fmaxf(v0, v1)));
      const float p0 = exp2f(v0 - mnew), p1 = exp2f(v1 - mnew);
      S[hh * kTK + lane] = p0;
      S[hh * kTK + lane + 32] = p1;
      const float sum = warp_sum(p0 + p1);
      if (lane == 0) {
        const float alpha = exp2f(mold - mnew);
        ls[hh] = ls[hh] * alpha + sum;
        ms[hh] = mnew;
        al[hh] = alpha;
      }
    }
    __syncthreads();
    if (2 * dp < HD) {  // o_h += P[h, :] . V
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int hh = hp + 2 * i;
        if (hh < G) {
          acc[i][0] *= al[hh];
          acc[i][1] *= al[hh];
        }
      }
      for (int j = 0; j < jn; ++j) {
        float v0, v1;
        if (sizeof(T) == 2) {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(Vt + (size_t)j * ROWP + 4 * dp);
          v0 = __uint_as_float(w << 16);
          v1 = __uint_as_float(w & 0xffff0000u);
        } else {
          const float2 f = *reinterpret_cast<const float2*>(Vt + (size_t)j * ROWP + 8 * dp);
          v0 = f.x;
          v1 = f.y;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int hh = hp + 2 * i;
          if (hh < G) {
            const float p = S[hh * kTK + j];
            acc[i][0] = fmaf(p, v0, acc[i][0]);
            acc[i][1] = fmaf(p, v1, acc[i][1]);
          }
        }
      }
    }
    __syncthreads();
  }

  if (2 * dp < HD) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int hh = hp + 2 * i;
      if (hh >= G) continue;
      const int h = g * G + hh;
      if (direct) {
        const float inv = 1.f / ls[hh];
        T* o = reinterpret_cast<T*>(a.out) + (size_t)r * a.out_row_stride + (size_t)h * HD + 2 * dp;
        o[0] = from_f<T>(acc[i][0] * inv);
        o[1] = from_f<T>(acc[i][1] * inv);
      } else {
        const size_t pidx = ((size_t)r * a.nh + h) * nsplit + split;
        float* po = part_o + pidx * HD + 2 * dp;
        po[0] = acc[i][0];
        po[1] = acc[i][1];
      }
    }
  }
  if (!direct && tid < G) {
    const size_t pidx = ((size_t)r * a.nh + g * G + tid) * nsplit + split;
    part_ml[2 * pidx] = ms[tid];
    part_ml[2 * pidx + 1] = ls[tid];
  }
}

// Merge the splits of one (row, head): o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
template <typename T>
__global__ void attn_combine_kernel(AttnRows a, int nsplit, const float* part_o,
                                    const float* part_ml) {
  pdl_launch_dependents();
  pdl_wait();
  const int h = blockIdx.x, r = blockIdx.y, d = threadIdx.x;
  const size_t base = ((size_t)r * a.nh + h) * nsplit;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[2 * (base + s)]);
  float den = 0.f, o = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float m = part_ml[2 * (base + s)];
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    den = fmaf(part_ml[2 * (base + s) + 1], w, den);
    o = fmaf(part_o[(base + s) * a.hd + d], w, o);
  }
  T* out = reinterpret_cast<T*>(a.out) + (size_t)r * a.out_row_stride + (size_t)h * a.hd;
  out[d] = from_f<T>(den > 0.f ? o / den : 0.f);
}

// Prefill attention implementation: 0 the tcgen05 kernel (default), 1 the
// mma.sync kernel (Q2_PREFILL_ATTN=mma selects it, for comparisons).
int prefill_attn_impl() {
  static const int v = [] {
    const char* e = getenv("Q2_PREFILL_ATTN");
    return (e && std::string(e) == "mma") ? 1 : 0;
  }();
  return v;
}

int attn_splits(int rows, int nkv, int max_keys) {
  long long ctas = (long long)rows * nkv;
  // as many splits as fit one wave of two CTAs per SM (a partial second wave
  // would leave most SMs idle for its duration); at least one
  long long want = (2LL * num_sms()) / (ctas ? ctas : 1);
  long long cap = (max_keys + kTK - 1) / kTK;
  if (cap > 64) cap = 64;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return (int)want;
}

size_t attn_scratch_bytes(int rows, int nh, int hd, int nsplit) {
  if (nsplit <= 1) return 0;
  size_t n = (size_t)rows * nh * nsplit;
  return n * hd * sizeof(float) + 2 * n * sizeof(float) + 256;
}

template <typename T, int HD>
static q2_status attn_t(const AttnRows& a, int nsplit, void* scratch, cudaStream_t st, bool pdl) {
  const size_t smem = AttnSmem<T, HD>::kBytes;
  Q2_CUDA_TRY(cudaFuncSetAttribute(attn_split_kernel<T, HD>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  float* po = nullptr;
  float* pml = nullptr;
  if (nsplit > 1) {
    po = reinterpret_cast<float*>(scratch);
    pml = po + (size_t)a.rows * a.nh * nsplit * HD;
  }
  Q2_LAUNCH(attn_split_kernel<T, HD>, dim3(nsplit, a.nkv, a.rows), dim3(kThreads), smem, st, pdl,
            a, nsplit, po, pml);
  if (nsplit > 1)
    Q2_LAUNCH(attn_combine_kernel<T>, dim3(a.nh, a.rows), dim3(HD), 0, st, pdl, a, nsplit,
              (const float*)po, (const float*)pml);
  return Q2_OK;
}

q2_status launch_attention(const AttnRows& a, int nsplit, void* scratch, int dtype,
                           cudaStream_t st, bool pdl, int* err, void* tc_ws) {
  if (attn_tc_supported(a, dtype) && prefill_attn_impl() == 0) {
    int* e = err ? err : op_error_flag();
    if (!e) {
      set_error("attention: no error word");
      return Q2_ERR_CUDA;
    }
    return launch_attn_tc(a, tc_ws, e, st);
  }
  if (attn_prefill_mma_supported(a, dtype)) return launch_attn_prefill_mma(a, st, pdl);
  if (a.rows == 0) return Q2_OK;
  if (a.nkv <= 0 || a.nh % a.nkv != 0 || a.nh / a.nkv > kGMax) {
    set_error("attention: need nh % nkv == 0 and nh / nkv <= 8");
    return Q2_ERR_SHAPE;
  }
  if (nsplit > 1 && !scratch) {
    set_error("attention: split partials need scratch memory");
    return Q2_ERR_INVALID_ARG;
  }
  const bool bf = dtype == Q2_BF16;
  switch (a.hd) {
    case 32: return bf ? attn_t<__nv_bfloat16, 32>(a, nsplit, scratch, st, pdl)
                       : attn_t<float, 32>(a, nsplit, scratch, st, pdl);
    case 64: return bf ? attn_t<__nv_bfloat16, 64>(a, nsplit, scratch, st, pdl)
                       : attn_t<float, 64>(a, nsplit, scratch, st, pdl);
    case 128: return bf ? attn_t<__nv_bfloat16, 128>(a, nsplit, scratch, st, pdl)
                        : attn_t<float, 128>(a, nsplit, scratch, st, pdl);
    default: set_error("attention: head_dim must be 32, 64 or 128"); return Q2_ERR_SHAPE;
  }
}

}  // namespace q2
