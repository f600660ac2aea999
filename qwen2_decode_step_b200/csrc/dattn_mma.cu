// dattn_mma.cu -- decode attention over the KV cache on the tensor cores.
//
// One CTA per (split of the visible keys, kv head, sequence), four warps.
// K/V tiles of 64 positions x 128 dims arrive by TMA (two 64-column boxes
// each, 128-byte swizzle) into a two-stage ring; warp w takes keys
// [16w, 16w + 16) of every tile:
//   scores  S[h][j] = q_h . k_j      mma.sync m16n8k16, the kv head's query
//                                    heads on M (rows >= G are zero), keys
//                                    on N, head dims on K; K fragments by
//                                    ldmatrix from the swizzled tile
//   softmax online per warp in fp32 (exp2 with scale * log2(e) applied to
//           the fp32 scores), the running max and sum held per head
//   output  O[h][d] += P[h][j] v_j[d] mma.sync with P as A, straight from the
//                                    score registers (split into a bf16 high
//                                    and low part, two MMAs), and V
//                                    fragments by ldmatrix.trans
// The four warps' (max, sum, unnormalised output) are merged in shared
// memory, each split writes its partial, and the last split of a (sequence,
// kv head) to finish merges all partials in split order (bit-reproducible),
// writing the attention output in bf16.
//
// Definition followed: the attention of the Day-0 adaptation tutorial (step
// 5): scores q k^T * scale with the causal mask (here: every cached position
// up to and including the new token), stable softmax, times V.
#include "common.cuh"
#include "decode.h"
#include "tma.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kMT = 64;          // keys per tile
constexpr int kMThreads = 128;   // four warps
constexpr int kMHD = 128;        // head dim of this kernel
constexpr int kMGMax = 8;        // query heads per kv head
constexpr int kMSplitMax = 64;
constexpr uint32_t kMWaitLimit = 1u << 22;
constexpr float kMLog2e = 1.4426950408889634f;

struct MSmem {
  static constexpr size_t kTile = (size_t)kMT * kMHD * 2;  // one K (or V) tile, 16 KB
  static constexpr size_t kO = 4 * kTile;                   // after [2 stages][K | V]
  static constexpr size_t kML = kO + 4 * (size_t)kMGMax * kMHD * 4;
  static constexpr size_t kW = kML + 4 * (size_t)kMGMax * 2 * 4;
  static constexpr size_t kBars = kW + 2 * (size_t)kMGMax * kMSplitMax * 4;
  static constexpr size_t kFlag = kBars + 2 * 8;
  static constexpr size_t kTotal = kFlag + 16 + 1024;  // + slack to align the base to 1024 B
};

// Byte offset of (row r, column c) in a 64 x 64 bf16 box laid down by TMA with
// 128-byte swizzle: 16-byte chunk c/8 of row r sits at chunk (c/8) ^ (r % 8).
__device__ __forceinline__ uint32_t swz_off(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7)) << 4) | ((c & 7) << 1)));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// c += A . B for one m16n8k16 tile (bf16 in, fp32 accumulate); A rows 8..15 are
// zero, so only a0 (row g, k pair 2t) and a2 (row g, k pair 2t + 8) are given.
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

}  // namespace

__global__ void __launch_bounds__(kMThreads) dattn_mma_kernel(const DAttn a,
                                                              const __grid_constant__ CUtensorMap kmap,
                                                              const __grid_constant__ CUtensorMap vmap) {
  using SM = MSmem;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* Ow = reinterpret_cast<float*>(smem + SM::kO);   // [4 warps][8 heads][128]
  float* MLw = reinterpret_cast<float*>(smem + SM::kML);  // [4 warps][8 heads][2]
  float* wts = reinterpret_cast<float*>(smem + SM::kW);   // [8][64] split weights
  float* mraw = wts + kMGMax * kMSplitMax;                 // [8][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBars);
  int& s_last = *reinterpret_cast<int*>(smem + SM::kFlag);

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = a.nh / a.nkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;  // mma fragment coordinates
  // Lengths change only at the end of a step, so they may be read before the
  // wait on the previous kernel.
  const int L = a.lens[b] + 1;
  const int ntiles = (L + kMT - 1) / kMT;
  const int active = min(a.nsplit, ntiles);
  const int tps = (ntiles + active - 1) / active;
  const int t0 = split * tps, t1 = min(t0 + tps, ntiles);
  const int row_base = ((a.layer * a.Bmax + b) * a.nkv + g) * a.max_seq;
  const int old_end = (L - 1) / kMT;  // tiles below hold only positions written by earlier steps

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int t, int stg) {
    uint8_t* kt = smem + (size_t)stg * 2 * SM::kTile;
    uint8_t* vt = kt + SM::kTile;
    mbar_arrive_expect_tx(&bars[stg], 2 * (uint32_t)SM::kTile);
#pragma unroll
    for (int bx = 0; bx < kMHD / 64; ++bx) {
      tma_load_2d(kt + bx * 8192, &kmap, bx * 64, row_base + t * kMT, &bars[stg]);
      tma_load_2d(vt + bx * 8192, &vmap, bx * 64, row_base + t * kMT, &bars[stg]);
    }
  };
  int pre = 0;
  if (tid == 0)
    for (; pre < 2 && t0 + pre < t1 && t0 + pre < old_end; ++pre) issue(t0 + pre, pre);
  pdl_launch_dependents();
  pdl_wait();
  if (tid == 0)
    for (int s = pre; s < 2 && t0 + s < t1; ++s) issue(t0 + s, s);

  // A fragments of the query heads (unscaled bf16): k-step kk covers dims
  // [16kk, 16kk + 16); rows gq >= G are zero.
  uint32_t qa[8][2];
  {
    const bf16* qrow = reinterpret_cast<const bf16*>(a.q) + (size_t)b * a.q_stride + (size_t)(g * G + gq) * kMHD;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qa[kk][0] = gq < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * tq) : 0u;
      qa[kk][1] = gq < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * tq + 8) : 0u;
    }
  }
  const float sl2 = a.scale * kMLog2e;
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: this lane addresses row mr of matrix mi

  for (int t = t0; t < t1; ++t) {
    const int stg = (t - t0) & 1;
    if (!mbar_wait(&bars[stg], (uint32_t)(((t - t0) >> 1) & 1), kMWaitLimit) && lane == 0)
      atomicOr(a.err, 2);
    const uint32_t kt = smem_u32(smem + (size_t)stg * 2 * SM::kTile);
    const uint32_t vt = kt + (uint32_t)SM::kTile;

    // ---- scores of this warp's 16 keys: s0 keys +0..7, s1 keys +8..15
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int key = warp * 16 + ((mi >> 1) << 3) + mr;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int dim = 16 * kk + ((mi & 1) << 3);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kt + (uint32_t)((dim >> 6) * 8192) + swz_off(key, dim & 63), r0, r1, r2, r3);
        mma16816(s0, qa[kk][0], qa[kk][1], r0, r1);
        mma16816(s1, qa[kk][0], qa[kk][1], r2, r3);
      }
    }
    // ---- online softmax for head gq over keys kb + 2tq, +1 and kb + 8 + 2tq, +1
    const int kb = t * kMT + warp * 16 + 2 * tq;
    float sc[4] = {s0[0] * sl2, s0[1] * sl2, s1[0] * sl2, s1[1] * sl2};
    if (kb >= L) sc[0] = -INFINITY;
    if (kb + 1 >= L) sc[1] = -INFINITY;
    if (kb + 8 >= L) sc[2] = -INFINITY;
    if (kb + 9 >= L) sc[3] = -INFINITY;
    float mloc = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const float mnew = fmaxf(m_run, mloc);
    const float msafe = mnew == -INFINITY ? 0.f : mnew;
    const float alpha = exp2f(m_run - msafe);
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = exp2f(sc[i] - msafe);
    float psum = (p[0] + p[1]) + (p[2] + p[3]);
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    l_run = l_run * alpha + psum;
    m_run = mnew;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= alpha;
      o[n][1] *= alpha;
    }
    // P in two bf16 parts, hi = bf16(p) and lo = bf16(p - hi), so that the
    // probabilities keep ~16 significant bits through the bf16 MMA (V is
    // exact in bf16; the products accumulate in fp32).
    float ph[4], pl[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ph[i] = __bfloat162float(__float2bfloat16_rn(p[i]));
      pl[i] = p[i] - ph[i];
    }
    const uint32_t pa0 = pack_bf16x2(ph[0], ph[1]), pa2 = pack_bf16x2(ph[2], ph[3]);
    const uint32_t pb0 = pack_bf16x2(pl[0], pl[1]), pb2 = pack_bf16x2(pl[2], pl[3]);
    // Positions past the sequence hold stale cache rows (possibly not finite):
    // their V entries are zeroed, as 0 * inf would poison the sum.  Lane (g, t)
    // holds V at the same keys kb, kb + 1 (b0) and kb + 8, kb + 9 (b1).
    const uint32_t vm0 = (kb < L ? 0x0000ffffu : 0u) | (kb + 1 < L ? 0xffff0000u : 0u);
    const uint32_t vm1 = (kb + 8 < L ? 0x0000ffffu : 0u) | (kb + 9 < L ? 0xffff0000u : 0u);

    // ---- O += P . V over the same 16 keys, 16 dims (two n8 tiles) per ldmatrix
    {
      const int key = warp * 16 + ((mi & 1) << 3) + mr;
#pragma unroll
      for (int nd = 0; nd < 8; ++nd) {
        const int dim = 16 * nd + ((mi >> 1) << 3);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(vt + (uint32_t)((dim >> 6) * 8192) + swz_off(key, dim & 63), r0, r1, r2, r3);
        r0 &= vm0;
        r1 &= vm1;
        r2 &= vm0;
        r3 &= vm1;
        mma16816(o[2 * nd], pa0, pa2, r0, r1);
        mma16816(o[2 * nd], pb0, pb2, r0, r1);
        mma16816(o[2 * nd + 1], pa0, pa2, r2, r3);
        mma16816(o[2 * nd + 1], pb0, pb2, r2, r3);
      }
    }
    __syncthreads();  // every warp is done with this stage
    if (tid == 0 && t + 2 < t1) issue(t + 2, stg);
  }

  // ---- merge the four warps: this split's (max, sum, unnormalised output)
  if (gq < G) {
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      float* dst = Ow + ((size_t)warp * kMGMax + gq) * kMHD + 8 * n + 2 * tq;
      dst[0] = o[n][0];
      dst[1] = o[n][1];
    }
    if (tq == 0) {
      MLw[(warp * kMGMax + gq) * 2] = m_run;
      MLw[(warp * kMGMax + gq) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  const bool direct = a.nsplit == 1;
  for (int i = tid; i < G * kMHD; i += kMThreads) {
    const int hh = i / kMHD, d = i % kMHD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, MLw[(w * kMGMax + hh) * 2]);
    const float Ms = M == -INFINITY ? 0.f : M;
    float O = 0.f, Lsum = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float e = exp2f(MLw[(w * kMGMax + hh) * 2] - Ms);
      O = fmaf(e, Ow[((size_t)w * kMGMax + hh) * kMHD + d], O);
      Lsum = fmaf(e, MLw[(w * kMGMax + hh) * 2 + 1], Lsum);
    }
    if (direct) {
      reinterpret_cast<bf16*>(a.out)[(size_t)b * a.nh * kMHD + (size_t)(g * G + hh) * kMHD + d] =
          from_f<bf16>(Lsum > 0.f ? O / Lsum : 0.f);
    } else {
      const size_t pidx = ((size_t)b * a.nh + g * G + hh) * a.nsplit + split;
      a.part_o[pidx * kMHD + d] = O;
      if (d == 0) {
        a.part_ml[2 * pidx] = M;
        a.part_ml[2 * pidx + 1] = Lsum;
      }
    }
  }
  if (direct) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counters + b * a.nkv + g, 1u) == (unsigned)a.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- the last split merges: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
  // over the splits that can hold keys (s < active), in split order.
  for (int i = tid; i < G * active; i += kMThreads) {
    const int hh = i / active, sp = i % active;
    const size_t pidx = ((size_t)b * a.nh + g * G + hh) * a.nsplit + sp;
    mraw[hh * kMSplitMax + sp] = __ldcg(a.part_ml + 2 * pidx);
    wts[hh * kMSplitMax + sp] = __ldcg(a.part_ml + 2 * pidx + 1);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int sp = 0; sp < active; ++sp) M = fmaxf(M, mraw[tid * kMSplitMax + sp]);
    const float Ms = M == -INFINITY ? 0.f : M;
    float den = 0.f;
    for (int sp = 0; sp < active; ++sp) {
      const float e = exp2f(mraw[tid * kMSplitMax + sp] - Ms);
      mraw[tid * kMSplitMax + sp] = e;
      den = fmaf(wts[tid * kMSplitMax + sp], e, den);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int sp = 0; sp < active; ++sp) wts[tid * kMSplitMax + sp] = mraw[tid * kMSplitMax + sp] * inv;
  }
  __syncthreads();
  for (int i = tid; i < G * kMHD; i += kMThreads) {
    const int hh = i / kMHD, d = i % kMHD;
    const size_t base = ((size_t)b * a.nh + g * G + hh) * a.nsplit;
    float acc = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < active; ++sp)
      acc = fmaf(wts[hh * kMSplitMax + sp], __ldcg(a.part_o + (base + sp) * kMHD + d), acc);
    reinterpret_cast<bf16*>(a.out)[(size_t)b * a.nh * kMHD + (size_t)(g * G + hh) * kMHD + d] =
        from_f<bf16>(acc);
  }
  if (tid == 0) a.counters[b * a.nkv + g] = 0u;
}

bool dattn_mma_supported(int nh, int nkv, int hd, int nsplit) {
  return hd == kMHD && nkv > 0 && nh % nkv == 0 && nh / nkv <= kMGMax && nsplit >= 1 &&
         nsplit <= kMSplitMax;
}

q2_status launch_dattn_mma(const DAttn& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                           cudaStream_t st) {
  if (!dattn_mma_supported(a.nh, a.nkv, a.hd, a.nsplit)) {
    set_error("decode attention (tensor cores): unsupported shape");
    return Q2_ERR_SHAPE;
  }
  const size_t smem = MSmem::kTotal;
  Q2_CUDA_TRY(cudaFuncSetAttribute(dattn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  Q2_LAUNCH(dattn_mma_kernel, dim3(a.nsplit, a.nkv, a.B), dim3(kMThreads), smem, st, true, a, kmap, vmap);
  return Q2_OK;
}

}  // namespace q2
