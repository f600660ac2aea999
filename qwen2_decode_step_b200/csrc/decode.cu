// decode.cu -- fused bf16 decode-step kernels (see decode.h).
//
// Numerics follow the operator boundaries of the model: every value that an
// operator writes back is rounded to bf16 exactly where the operator would
// round it (linear outputs, RoPE outputs, the RMSNorm output, the SwiGLU
// output, each residual add), even when the next operator consumes it inside
// the same kernel.
#include <limits.h>

#include "common.cuh"
#include "decode.h"
#include "tma.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

// Warp roles: kConsumers warps compute, one producer warp streams weights.
constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr size_t kRingBytes = 96 * 1024;
constexpr uint32_t kWaitLimit = 1u << 22;

struct Geo {
  int rows_per_stage;  // whole weight rows per ring slot (even for paired epilogues)
  int rows_per_unit;   // 2 for the paired epilogues (RoPE pair, gate/up pair), else 1
  int stage_bytes;
  int stages_total;
  int grid;
  int ring;            // ring slots
};

struct Lay {
  size_t act, full, empty, am_i, am_v, flag, total;
};

__host__ __device__ inline size_t up16(size_t v) { return (v + 15) & ~(size_t)15; }

__host__ __device__ inline Lay layout(const Geo& g, int K, int mt) {
  Lay L;
  size_t o = (size_t)g.ring * g.stage_bytes;
  L.act = o;
  o = up16(o + (size_t)mt * K * 2);
  L.full = o;
  o += (size_t)g.ring * 8;
  L.empty = o;
  o = up16(o + (size_t)g.ring * 8);
  L.am_i = o;
  o += kConsumers * 4 * sizeof(long long);
  L.am_v = o;
  o += kConsumers * 4 * sizeof(float);
  L.flag = o;
  L.total = up16(o + 16);
  return L;
}

Geo geometry(int epi, int N, int K) {
  Geo g;
  const int row_bytes = K * 2;
  g.rows_per_unit = (epi == EPI_QKV || epi == EPI_SWIGLU) ? 2 : 1;
  int r = 8;
  while (r > g.rows_per_unit && (size_t)r * row_bytes > 24 * 1024) r >>= 1;
  g.rows_per_stage = r;
  g.stage_bytes = r * row_bytes;
  g.stages_total = (N + r - 1) / r;
  g.grid = g.stages_total < num_sms() ? g.stages_total : num_sms();
  const int per_cta = (g.stages_total + g.grid - 1) / g.grid;
  // A parity wait on an mbarrier only tells the current phase from the next
  // one, so no consumer may wait for use k+1 of a slot before use k has
  // completed.  Stage s goes to warps (s*units + u) % kConsumers: when slots
  // are reused, ring * units must be a multiple of kConsumers so that the
  // same warps consume every use of a slot, in order.  A ring at least as
  // deep as the CTA's stage count uses every slot once.
  const int units = g.rows_per_stage / g.rows_per_unit;
  int q = 1;  // the smallest ring step with q * units a multiple of kConsumers
  while ((q * units) % kConsumers != 0) ++q;
  int ring = (int)(kRingBytes / g.stage_bytes);
  ring = ring / q * q;
  if (ring < q) ring = q;
  if (ring >= per_cta) ring = per_cta;
  g.ring = ring;
  return g;
}

__device__ __forceinline__ float silu_mul(float gv, float uv) {
  return uv * (gv / (1.0f + expf(-gv)));
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

}  // namespace

// ---------------------------------------------------------------- dgemv
// NCH > 0: K == NCH * 256 and the single token's activation stays in
// registers (each lane keeps its NCH 8-element chunks, unpacked to fp32);
// NCH == 0: the activation is read from shared memory per chunk.
template <int EPI, int MT, int NCH>
__global__ void __launch_bounds__(kThreads, 1) dgemv_kernel(const DGemv a, const Geo g) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const Lay L = layout(g, a.K, MT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  uint8_t* ring = smem;
  bf16* act = reinterpret_cast<bf16*>(smem + L.act);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.empty);

  const int s_begin = (int)((long long)blockIdx.x * g.stages_total / g.grid);
  const int s_end = (int)((long long)(blockIdx.x + 1) * g.stages_total / g.grid);
  const int ns = s_end - s_begin;
  const int units = g.rows_per_stage / g.rows_per_unit;  // work units per stage

  if (tid == 0) {
    for (int i = 0; i < g.ring; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], units);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // ---------------- producer warp: weights do not depend on the previous
  // kernel, so it streams without waiting for it.
  if (warp == kConsumers) {
    if (lane == 0) {
      const bf16* w = reinterpret_cast<const bf16*>(a.w);
      const uint64_t pol = policy_evict_first();
      for (int s = 0; s < ns; ++s) {
        const int slot = s % g.ring;
        if (s >= g.ring && !mbar_wait(&empty[slot], (uint32_t)(((s / g.ring) - 1) & 1), kWaitLimit))
          atomicOr(a.err, 2);
        const int row0 = (s_begin + s) * g.rows_per_stage;
        const int rows = min(g.rows_per_stage, a.N - row0);
        const uint32_t bytes = (uint32_t)rows * K * 2;
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s_evict_first(ring + (size_t)slot * g.stage_bytes, w + (size_t)row0 * K, bytes,
                             &full[slot], pol);
      }
    }
    return;
  }

  // ---------------- consumer warps
  pdl_wait();
  const bf16* x = reinterpret_cast<const bf16*>(a.x);
  const int ct = tid;  // consumer thread index, 0 .. kConsumers*32-1
  if (a.norm_w) {  // act[m] = rmsnorm(x[m]) * norm_w, one rounding
    const bf16* nw = reinterpret_cast<const bf16*>(a.norm_w);
    float* red = reinterpret_cast<float*>(smem + L.am_v);  // borrowed: [kConsumers][MT]
    float ss[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) ss[m] = 0.f;
    for (int k = ct * 8; k < K; k += kConsumers * 32 * 8) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < a.M) {
          float f[8];
          unpack16<bf16>(*reinterpret_cast<const uint4*>(x + (size_t)m * K + k), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss[m] = fmaf(f[e], f[e], ss[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float v = warp_sum(ss[m]);
      if (lane == 0) red[warp * MT + m] = v;
    }
    consumer_sync();
    float inv[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < kConsumers; ++i) t += red[i * MT + m];
      inv[m] = rsqrtf(t / (float)K + a.eps);
    }
    for (int k = ct * 8; k < K; k += kConsumers * 32 * 8) {
      float wf[8];
      unpack16<bf16>(*reinterpret_cast<const uint4*>(nw + k), wf);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < a.M) {
          float f[8];
          unpack16<bf16>(*reinterpret_cast<const uint4*>(x + (size_t)m * K + k), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = f[e] * inv[m] * wf[e];
          *reinterpret_cast<uint4*>(act + (size_t)m * K + k) = pack16<bf16>(f);
        }
      }
    }
  } else {
    for (int k = ct * 8; k < K; k += kConsumers * 32 * 8) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < a.M)
          *reinterpret_cast<uint4*>(act + (size_t)m * K + k) =
              *reinterpret_cast<const uint4*>(x + (size_t)m * K + k);
    }
  }
  consumer_sync();

  // Register copy of the activation (NCH > 0): lane's chunks lane + 32*i.
  float xr[NCH > 0 ? NCH : 1][8];
  if (NCH > 0) {
#pragma unroll
    for (int i = 0; i < (NCH > 0 ? NCH : 1); ++i)
      unpack16<bf16>(reinterpret_cast<const uint4*>(act)[lane + 32 * i], xr[i]);
  }

  float best_v = -INFINITY;  // EPI_LOGITS: lane m < MT tracks token m
  long long best_i = LLONG_MAX;
  const int nch = K / 8;

  // Work item i = s * units + u goes to consumer warp i % kConsumers.
  for (int item = warp; item < ns * units; item += kConsumers) {
    const int s = item / units, u = item % units;
    const int slot = s % g.ring;
    if (!mbar_wait(&full[slot], (uint32_t)((s / g.ring) & 1), kWaitLimit) && lane == 0)
      atomicOr(a.err, 2);
    const uint8_t* stg = ring + (size_t)slot * g.stage_bytes;
    const int row0 = (s_begin + s) * g.rows_per_stage;
    const int rows = min(g.rows_per_stage, a.N - row0);
    float y[2][MT];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) y[r][m] = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r >= g.rows_per_unit) break;
      const int rr = u * g.rows_per_unit + r;
      if (rr >= rows) break;
      const uint4* wrow = reinterpret_cast<const uint4*>(stg + (size_t)rr * K * 2);
      if (NCH > 0) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < (NCH > 0 ? NCH : 1); ++i) {
          float wf[8];
          unpack16<bf16>(wrow[lane + 32 * i], wf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e & 3] = fmaf(wf[e], xr[i][e], acc[e & 3]);
        }
        y[r][0] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      } else {
        float acc[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = 0.f;
#pragma unroll 4
        for (int c = lane; c < nch; c += 32) {
          float wf[8];
          unpack16<bf16>(wrow[c], wf);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < a.M) {
              float xf[8];
              unpack16<bf16>(reinterpret_cast<const uint4*>(act + (size_t)m * K)[c], xf);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[m][e & 1] = fmaf(wf[e], xf[e], acc[m][e & 1]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) y[r][m] = acc[m][0] + acc[m][1];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);  // this unit's rows are read
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) y[r][m] = warp_sum(y[r][m]);

    // ---- epilogue: lane m finishes token m of this unit
    const int m = lane;
    if (m < a.M && m < MT) {
      float y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int mm = 0; mm < MT; ++mm)
        if (mm == m) {
          y0 = y[0][mm];
          y1 = y[1][mm];
        }
      const int n0 = row0 + u * g.rows_per_unit;
      if (EPI == EPI_RESID) {
        if (n0 < a.N) {
          bf16* xo = reinterpret_cast<bf16*>(a.out) + (size_t)m * a.out_stride + n0;
          *xo = from_f<bf16>(to_f(*xo) + round_st<bf16>(y0));
        }
      } else if (EPI == EPI_SWIGLU) {
        if (n0 + 1 < a.N) {
          const float gv = round_st<bf16>(y0), uv = round_st<bf16>(y1);
          reinterpret_cast<bf16*>(a.out)[(size_t)m * a.out_stride + (n0 >> 1)] = from_f<bf16>(silu_mul(gv, uv));
        }
      } else if (EPI == EPI_QKV) {
        if (n0 + 1 < a.N) {
          const int hs = n0 / a.hd, j = (n0 % a.hd) >> 1, half = a.hd >> 1;
          const bf16* bias = reinterpret_cast<const bf16*>(a.bias);
          const float va = round_st<bf16>(y0 + to_f(bias[n0]));
          const float vb = round_st<bf16>(y1 + to_f(bias[n0 + 1]));
          const int pos = a.lens[m];
          if (hs < a.nh + a.nkv) {
            const float2 cs = a.rope[(size_t)pos * half + j];
            const bf16 ra = from_f<bf16>(va * cs.x - vb * cs.y);
            const bf16 rb = from_f<bf16>(vb * cs.x + va * cs.y);
            bf16* dst = hs < a.nh ? reinterpret_cast<bf16*>(a.out) + (size_t)m * a.out_stride + (size_t)hs * a.hd
                                  : reinterpret_cast<bf16*>(a.kc) + (size_t)m * a.kv_seq_stride +
                                        ((size_t)(hs - a.nh) * a.max_seq + pos) * a.hd;
            dst[j] = ra;
            dst[j + half] = rb;
          } else {
            bf16* vr = reinterpret_cast<bf16*>(a.vc) + (size_t)m * a.kv_seq_stride +
                       ((size_t)(hs - a.nh - a.nkv) * a.max_seq + pos) * a.hd;
            vr[j] = from_f<bf16>(va);
            vr[j + half] = from_f<bf16>(vb);
          }
        }
      } else {  // EPI_LOGITS
        if (n0 < a.N) {
          a.logits[(size_t)m * a.N + n0] = y0;
          if (am_better(y0, n0, best_v, best_i)) {
            best_v = y0;
            best_i = n0;
          }
        }
      }
    }
  }

  if (EPI == EPI_LOGITS) {
    long long* ami = reinterpret_cast<long long*>(smem + L.am_i);
    float* amv = reinterpret_cast<float*>(smem + L.am_v);
    int& s_last = *reinterpret_cast<int*>(smem + L.flag);
    if (lane < MT) {
      ami[warp * 4 + lane] = best_i;
      amv[warp * 4 + lane] = best_v;
    }
    consumer_sync();
    if (ct < a.M) {
      float bv = -INFINITY;
      long long bi = LLONG_MAX;
      for (int wv = 0; wv < kConsumers; ++wv)
        if (am_better(amv[wv * 4 + ct], ami[wv * 4 + ct], bv, bi)) {
          bv = amv[wv * 4 + ct];
          bi = ami[wv * 4 + ct];
        }
      a.am_val[blockIdx.x * kDecodeMaxBatch + ct] = bv;
      a.am_idx[blockIdx.x * kDecodeMaxBatch + ct] = bi;
    }
    __threadfence();
    consumer_sync();
    if (ct == 0) s_last = (atomicAdd(a.counter, 1u) == gridDim.x - 1);
    consumer_sync();
    if (s_last) {
      __threadfence();
      if (ct < a.M) {
        float bv = -INFINITY;
        long long bi = LLONG_MAX;
        for (unsigned b = 0; b < gridDim.x; ++b) {
          const float v = __ldcg(a.am_val + b * kDecodeMaxBatch + ct);
          const long long i = __ldcg(reinterpret_cast<const long long*>(a.am_idx) + b * kDecodeMaxBatch + ct);
          if (am_better(v, i, bv, bi)) {
            bv = v;
            bi = i;
          }
        }
        a.next[ct] = bi;
        if (a.lens_inc) a.lens_inc[ct] += 1;
      }
      if (ct == 0) *a.counter = 0u;
    }
  }
}

bool dgemv_supported(int epi, int N, int K) {
  if (K % 8 != 0 || N <= 0) return false;
  const Geo g = geometry(epi, N, K);
  if (g.rows_per_unit == 2 && (N % 2 != 0 || g.rows_per_stage % 2 != 0)) return false;
  if (g.stage_bytes > 64 * 1024) return false;
  return layout(g, K, kDecodeMaxBatch).total <= 220 * 1024;
}

int dgemv_grid(int epi, int N, int K) { return geometry(epi, N, K).grid; }

template <int EPI, int MT, int NCH>
static q2_status dgemv_launch(const DGemv& a, const Geo& g, cudaStream_t st) {
  const size_t smem = layout(g, a.K, MT).total;
  Q2_CUDA_TRY(cudaFuncSetAttribute(dgemv_kernel<EPI, MT, NCH>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  Q2_LAUNCH(dgemv_kernel<EPI, MT, NCH>, dim3(g.grid), dim3(kThreads), smem, st, true, a, g);
  return Q2_OK;
}

template <int EPI>
static q2_status dgemv_mt(const DGemv& a, const Geo& g, cudaStream_t st) {
  if (a.M <= 1) {
    if (a.K == 6 * 256) return dgemv_launch<EPI, 1, 6>(a, g, st);
    return dgemv_launch<EPI, 1, 0>(a, g, st);
  }
  if (a.M <= 2) return dgemv_launch<EPI, 2, 0>(a, g, st);
  return dgemv_launch<EPI, 4, 0>(a, g, st);
}

q2_status launch_dgemv(int epi, const DGemv& a, cudaStream_t st) {
  if (a.M < 1 || a.M > kDecodeMaxBatch || !dgemv_supported(epi, a.N, a.K)) {
    set_error("decode gemv: unsupported shape");
    return Q2_ERR_SHAPE;
  }
  const Geo g = geometry(epi, a.N, a.K);
  switch (epi) {
    case EPI_QKV: return dgemv_mt<EPI_QKV>(a, g, st);
    case EPI_RESID: return dgemv_mt<EPI_RESID>(a, g, st);
    case EPI_SWIGLU: return dgemv_mt<EPI_SWIGLU>(a, g, st);
    default: return dgemv_mt<EPI_LOGITS>(a, g, st);
  }
}

// ------------------------------------------------------------------ dattn
namespace {
constexpr int kAT = 64;        // keys per tile
constexpr int kAThreads = 128;
constexpr int kAGMax = 8;
constexpr float kLog2e = 1.4426950408889634f;

template <int HD>
struct ASmem {
  static constexpr int kTile = kAT * HD * 2;  // bytes of one K (or V) tile
  static constexpr size_t kQ = 4 * (size_t)kTile;
  static constexpr size_t kS = kQ + kAGMax * HD * 4;
  static constexpr size_t kM = kS + kAGMax * kAT * 4;
  static constexpr size_t kBars = kM + 3 * kAGMax * 4;
  static constexpr size_t kFlag = kBars + 2 * 8;
  static constexpr size_t kTotal = kFlag + 16 + 1024;  // + slack to align the base to 1024 B
};

// Byte offset of element (row r, column c) of a [64 rows][64 cols] bf16 box
// written by TMA with 128-byte swizzle: 16-byte chunk c/8 of row r lives at
// chunk position (c/8) ^ (r % 8) of that row.
__device__ __forceinline__ int swz(int r, int c) {
  return r * 128 + ((((c >> 3) ^ (r & 7)) << 4) | ((c & 7) << 1));
}
}  // namespace

template <int HD>
__global__ void __launch_bounds__(kAThreads) dattn_kernel(const DAttn a,
                                                          const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap) {
  using SM = ASmem<HD>;
  constexpr int NBOX = HD / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte-swizzled TMA boxes must start on 1024-byte boundaries for the
  // swizzle pattern (a function of the shared-memory address) to match swz().
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* qs = reinterpret_cast<float*>(smem + SM::kQ);
  float* S = reinterpret_cast<float*>(smem + SM::kS);
  float* ms = reinterpret_cast<float*>(smem + SM::kM);
  float* ls = ms + kAGMax;
  float* al = ls + kAGMax;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBars);
  int& s_last = *reinterpret_cast<int*>(smem + SM::kFlag);

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = a.nh / a.nkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // Lengths change only at the end of a step (the lm_head kernel), so they
  // can be read before waiting on the previous kernel.
  const int L = a.lens[b] + 1;
  const int ntiles = (L + kAT - 1) / kAT;
  const int active = min(a.nsplit, ntiles);
  const int tps = (ntiles + active - 1) / active;
  const int t0 = split * tps, t1 = min(t0 + tps, ntiles);
  const int row_base = ((a.layer * a.Bmax + b) * a.nkv + g) * a.max_seq;
  const int old_end = (L - 1) / kAT;  // tiles below hold only positions written by earlier steps

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int t, int stg) {
    uint8_t* kt = smem + (size_t)stg * 2 * SM::kTile;
    uint8_t* vt = kt + SM::kTile;
    mbar_arrive_expect_tx(&bars[stg], 2 * SM::kTile);
#pragma unroll
    for (int bx = 0; bx < NBOX; ++bx) {
      tma_load_2d(kt + bx * 8192, &kmap, bx * 64, row_base + t * kAT, &bars[stg]);
      tma_load_2d(vt + bx * 8192, &vmap, bx * 64, row_base + t * kAT, &bars[stg]);
    }
  };
  int pre = 0;
  if (tid == 0)
    for (; pre < 2 && t0 + pre < t1 && t0 + pre < old_end; ++pre) issue(t0 + pre, pre);
  pdl_launch_dependents();
  pdl_wait();
  if (tid == 0)
    for (int s = pre; s < 2 && t0 + s < t1; ++s) issue(t0 + s, s);

  const bf16* qrow = reinterpret_cast<const bf16*>(a.q) + (size_t)b * a.q_stride + (size_t)g * G * HD;
  const float qscale = a.scale * kLog2e;
  for (int i = tid; i < G * HD; i += kAThreads) qs[i] = to_f(qrow[i]) * qscale;
  if (tid < kAGMax) {
    ms[tid] = -INFINITY;
    ls[tid] = 0.f;
  }
  __syncthreads();

  const int dp = tid & 63, hp = tid >> 6;  // PV: dims (2dp, 2dp+1), heads hp, hp+2, ...
  float acc[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.f;

  for (int t = t0; t < t1; ++t) {
    const int stg = (t - t0) & 1;
    if (!mbar_wait(&bars[stg], (uint32_t)(((t - t0) >> 1) & 1), kWaitLimit) && lane == 0)
      atomicOr(a.err, 2);
    const uint8_t* kt = smem + (size_t)stg * 2 * SM::kTile;
    const uint8_t* vt = kt + SM::kTile;
    const int jn = min(kAT, L - t * kAT);
    {  // scores: thread j = tid & 63 takes key j for heads hp, hp+2, ...
      const int j = tid & 63;
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int bx = 0; bx < NBOX; ++bx) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float kf[8];
          unpack16<bf16>(*reinterpret_cast<const uint4*>(kt + bx * 8192 + swz(j, c * 8)), kf);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int hh = hp + 2 * i;
            if (hh < G) {
              const float* qh = qs + hh * HD + bx * 64 + c * 8;
#pragma unroll
              for (int e = 0; e < 8; ++e) sc[i] = fmaf(qh[e], kf[e], sc[i]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int hh = hp + 2 * i;
        if (hh < G) S[hh * kAT + j] = (j < jn) ? sc[i] : -INFINITY;
      }
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += kAThreads / 32) {
      const float v0 = S[hh * kAT + lane], v1 = S[hh * kAT + lane + 32];
      const float mold = ms[hh];
      const float mnew = fmaxf(mold, warp_max(fmaxf(v0, v1)));
      const float p0 = exp2f(v0 - mnew), p1 = exp2f(v1 - mnew);
      S[hh * kAT + lane] = p0;
      S[hh * kAT + lane + 32] = p1;
      const float sum = warp_sum(p0 + p1);
      if (lane == 0) {
        const float alpha = exp2f(mold - mnew);
        ls[hh] = ls[hh] * alpha + sum;
        ms[hh] = mnew;
        al[hh] = alpha;
      }
    }
    __syncthreads();
    if (2 * dp < HD) {
      const int bx = (2 * dp) >> 6, cc = (2 * dp) & 63;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int hh = hp + 2 * i;
        if (hh < G) {
          acc[i][0] *= al[hh];
          acc[i][1] *= al[hh];
        }
      }
      for (int j = 0; j < jn; ++j) {
        const uint32_t wv = *reinterpret_cast<const uint32_t*>(vt + bx * 8192 + swz(j, cc));
        const float v0 = __uint_as_float(wv << 16), v1 = __uint_as_float(wv & 0xffff0000u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int hh = hp + 2 * i;
          if (hh < G) {
            const float p = S[hh * kAT + j];
            acc[i][0] = fmaf(p, v0, acc[i][0]);
            acc[i][1] = fmaf(p, v1, acc[i][1]);
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0 && t + 2 < t1) issue(t + 2, stg);
  }

  // ---- partials of this split, then the last split of (b, g) merges them
  if (2 * dp < HD) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int hh = hp + 2 * i;
      if (hh < G) {
        const size_t pidx = ((size_t)b * a.nh + g * G + hh) * a.nsplit + split;
        a.part_o[pidx * HD + 2 * dp] = acc[i][0];
        a.part_o[pidx * HD + 2 * dp + 1] = acc[i][1];
      }
    }
  }
  if (tid < G) {
    const size_t pidx = ((size_t)b * a.nh + g * G + tid) * a.nsplit + split;
    const bool empty = t0 >= t1;
    a.part_ml[2 * pidx] = empty ? -INFINITY : ms[tid];
    a.part_ml[2 * pidx + 1] = empty ? 0.f : ls[tid];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counters + b * a.nkv + g, 1u) == (unsigned)a.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // Merge: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the splits
  // that can hold keys (s < active; later ones are empty by construction).
  // The per-split weights go to shared memory first so that the output loop
  // below issues independent loads.
  float* wts = S;    // [G][active] (active <= 64 = kAT)
  float* mraw = qs;  // [G][active]
  for (int i = tid; i < G * active; i += kAThreads) {
    const int hh = i / active, sp = i % active;
    const size_t pidx = ((size_t)b * a.nh + g * G + hh) * a.nsplit + sp;
    mraw[i] = __ldcg(a.part_ml + 2 * pidx);
    wts[i] = __ldcg(a.part_ml + 2 * pidx + 1);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int sp = 0; sp < active; ++sp) M = fmaxf(M, mraw[tid * active + sp]);
    float den = 0.f;
    for (int sp = 0; sp < active; ++sp) {
      const float m = mraw[tid * active + sp];
      const float e = m == -INFINITY ? 0.f : exp2f(m - M);
      mraw[tid * active + sp] = e;
      den = fmaf(wts[tid * active + sp], e, den);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int sp = 0; sp < active; ++sp) wts[tid * active + sp] = mraw[tid * active + sp] * inv;
  }
  __syncthreads();
  for (int i = tid; i < G * HD; i += kAThreads) {
    const int hh = i / HD, d = i % HD;
    const size_t base = ((size_t)b * a.nh + g * G + hh) * a.nsplit;
    float o = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < active; ++sp)
      o = fmaf(wts[hh * active + sp], __ldcg(a.part_o + (base + sp) * HD + d), o);
    reinterpret_cast<bf16*>(a.out)[(size_t)b * a.nh * HD + (size_t)(g * G + hh) * HD + d] = from_f<bf16>(o);
  }
  if (tid == 0) a.counters[b * a.nkv + g] = 0u;
}

bool dattn_supported(int nh, int nkv, int hd) {
  return (hd == 64 || hd == 128) && nkv > 0 && nh % nkv == 0 && nh / nkv <= kAGMax;
}

q2_status launch_dattn(const DAttn& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t st) {
  if (!dattn_supported(a.nh, a.nkv, a.hd)) {
    set_error("decode attention: unsupported shape");
    return Q2_ERR_SHAPE;
  }
  dim3 grid(a.nsplit, a.nkv, a.B);
  if (a.hd == 128) {
    const size_t smem = ASmem<128>::kTotal;
    Q2_CUDA_TRY(cudaFuncSetAttribute(dattn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    Q2_LAUNCH(dattn_kernel<128>, grid, dim3(kAThreads), smem, st, true, a, kmap, vmap);
  } else {
    const size_t smem = ASmem<64>::kTotal;
    Q2_CUDA_TRY(cudaFuncSetAttribute(dattn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    Q2_LAUNCH(dattn_kernel<64>, grid, dim3(kAThreads), smem, st, true, a, kmap, vmap);
  }
  return Q2_OK;
}

}  // namespace q2
