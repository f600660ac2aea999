// attn_mma.cu -- causal GQA attention of a block of query rows of one
// sequence (prefill) on the tensor cores, flash-attention style.
//
// One CTA per (64 query rows, query head), four warps of 16 rows each.  The
// CTA stages its Q block once and then walks the visible keys in tiles of 64
// (K and V double-buffered with cp.async into 256-byte rows whose 16-byte
// chunks are XOR-swizzled by row, so ldmatrix reads are bank-conflict free):
//   S = Q K^T          mma.sync m16n8k16 (rows on M, keys on N, dims on K)
//   online softmax     fp32, exp2 with scale * log2(e) on the fp32 scores,
//                      causal mask on the diagonal tile
//   O += P V           P from the score registers in two bf16 parts (high and
//                      low, ~16 significant bits), V by ldmatrix.trans
// Output rows are normalised and written in bf16.
//
// Definition followed: the attention of the Day-0 adaptation tutorial (step
// 5): scores q k^T * scale, causal mask (query i of a block at positions
// p0.. sees keys j <= p0 + i), stable softmax, times V; query head h reads kv
// head h / (nh / nkv).
#include "common.cuh"
#include "kernels.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kPQ = 64;         // query rows per CTA
constexpr int kPK = 64;         // keys per tile
constexpr int kPHD = 128;       // head dim
constexpr int kPThreads = 128;  // four warps x 16 rows
constexpr float kPLog2e = 1.4426950408889634f;

struct PSmem {
  static constexpr size_t kTile = (size_t)kPK * kPHD * 2;  // 16 KB (also the Q block)
  static constexpr size_t kQ = 0;
  static constexpr size_t kK = kTile;            // [2][64][128]
  static constexpr size_t kV = kK + 2 * kTile;   // [2][64][128]
  static constexpr size_t kTotal = kV + 2 * kTile;
};

// Byte offset of 16-byte chunk c (0..15) of row r in a [rows][256 B] tile
// whose chunks are XOR-swizzled by (r % 8).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void p_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void p_ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// c += A . B, one m16n8k16 tile, bf16 operands, fp32 accumulators.
__device__ __forceinline__ void p_mma(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t p_pack(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

}  // namespace

__global__ void __launch_bounds__(kPThreads) attn_prefill_mma_kernel(const AttnRows a) {
  extern __shared__ __align__(128) uint8_t psm[];
  const uint32_t sQ = smem_u32(psm + PSmem::kQ);
  const uint32_t sK = smem_u32(psm + PSmem::kK);
  const uint32_t sV = smem_u32(psm + PSmem::kV);

  pdl_launch_dependents();
  pdl_wait();

  const int qb = blockIdx.x, h = blockIdx.y;
  const int G = a.nh / a.nkv, g = h / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int mi = lane >> 3, mr = lane & 7;
  const int r0 = qb * kPQ;                      // first query row of the block
  const int nrows = min(kPQ, a.rows - r0);
  const int seq = a.fixed_seq;
  // visible keys of row r: [0, base + row_step * r)
  const int vis_last = a.base + a.row_step * (r0 + nrows - 1);  // of the block's last row
  const int ntiles = (vis_last + kPK - 1) / kPK;

  const bf16* kbase = reinterpret_cast<const bf16*>(a.k) + (size_t)seq * a.kv_seq_stride + (size_t)g * a.kv_head_stride;
  const bf16* vbase = reinterpret_cast<const bf16*>(a.v) + (size_t)seq * a.kv_seq_stride + (size_t)g * a.kv_head_stride;

  // ---- Q block (rows past the end read as zeros)
  for (int c = tid; c < kPQ * 16; c += kPThreads) {
    const int r = c >> 4, ch = c & 15;
    const bool ok = r < nrows;
    const bf16* src = reinterpret_cast<const bf16*>(a.q) + (size_t)(r0 + (ok ? r : 0)) * a.q_row_stride +
                      (size_t)h * kPHD + ch * 8;
    cp_async16(psm + PSmem::kQ + sw_off(r, ch), src, ok);
  }
  auto issue = [&](int t, int buf) {
    const int j0 = t * kPK;
    for (int c = tid; c < kPK * 16; c += kPThreads) {
      const int r = c >> 4, ch = c & 15;
      const bool ok = j0 + r < vis_last;
      const size_t off = (size_t)(ok ? j0 + r : 0) * a.kv_tok_stride + ch * 8;
      cp_async16(psm + PSmem::kK + (size_t)buf * PSmem::kTile + sw_off(r, ch), kbase + off, ok);
      cp_async16(psm + PSmem::kV + (size_t)buf * PSmem::kTile + sw_off(r, ch), vbase + off, ok);
    }
  };
  issue(0, 0);
  cp_async_commit();

  const float sl2 = a.scale * kPLog2e;
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows gq, gq + 8
  uint32_t qa[8][4];
  const int wr = warp * 16;  // this warp's first row in the block
  // causal limit (exclusive) of this lane's two rows
  const int lim0 = a.base + a.row_step * (r0 + wr + gq);
  const int lim1 = a.base + a.row_step * (r0 + wr + gq + 8);

  for (int t = 0; t < ntiles; ++t) {
    const int buf = t & 1;
    if (t + 1 < ntiles) {
      issue(t + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {  // the Q block has landed: A fragments of this warp's 16 rows
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int row = wr + ((mi & 1) << 3) + mr, ch = 2 * kk + (mi >> 1);
        p_ldsm_x4(sQ + sw_off(row, ch), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    const uint32_t kt = sK + (uint32_t)(buf * PSmem::kTile), vt = sV + (uint32_t)(buf * PSmem::kTile);
    const int j0 = t * kPK;
    // a tile past every row of this warp contributes nothing (warp-uniform:
    // the MMAs and ldmatrix below are collective)
    const bool live = j0 < a.base + a.row_step * (r0 + wr + 15);

    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
    if (live) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {  // keys [16np, 16np + 16): two n8 tiles
          const int key = 16 * np + ((mi >> 1) << 3) + mr, ch = 2 * kk + (mi & 1);
          uint32_t b0, b1, b2, b3;
          p_ldsm_x4(kt + sw_off(key, ch), b0, b1, b2, b3);
          p_mma(s[2 * np], qa[kk], b0, b1);
          p_mma(s[2 * np + 1], qa[kk], b2, b3);
        }
      }
    }
    // ---- online softmax, rows gq (c0, c1) and gq + 8 (c2, c3)
    float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int j = j0 + 8 * n + 2 * tq;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[n][e] = (j + e < lim0) ? s[n][e] * sl2 : -INFINITY;
        s[n][2 + e] = (j + e < lim1) ? s[n][2 + e] * sl2 : -INFINITY;
        mt[0] = fmaxf(mt[0], s[n][e]);
        mt[1] = fmaxf(mt[1], s[n][2 + e]);
      }
    }
    float alpha[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mt[i] = fmaxf(mt[i], __shfl_xor_sync(0xffffffffu, mt[i], 1));
      mt[i] = fmaxf(mt[i], __shfl_xor_sync(0xffffffffu, mt[i], 2));
      const float mnew = fmaxf(m_run[i], mt[i]);
      const float msafe = mnew == -INFINITY ? 0.f : mnew;
      alpha[i] = exp2f(m_run[i] - msafe);
      m_run[i] = mnew;
      mt[i] = msafe;
    }
    float ps[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[n][e] = exp2f(s[n][e] - mt[0]);
        s[n][2 + e] = exp2f(s[n][2 + e] - mt[1]);
        ps[0] += s[n][e];
        ps[1] += s[n][2 + e];
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ps[i] += __shfl_xor_sync(0xffffffffu, ps[i], 1);
      ps[i] += __shfl_xor_sync(0xffffffffu, ps[i], 2);
      l_run[i] = l_run[i] * alpha[i] + ps[i];
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    if (live) {
      // ---- O += P V: k-step ks covers keys [16ks, 16ks + 16) = score tiles 2ks, 2ks + 1
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t ph[4], pl[4];
        float hv[8];
        const float* lo = s[2 * ks];
        const float* hi = s[2 * ks + 1];
        const float pv[8] = {lo[0], lo[1], lo[2], lo[3], hi[0], hi[1], hi[2], hi[3]};
#pragma unroll
        for (int i = 0; i < 8; ++i) hv[i] = __bfloat162float(__float2bfloat16_rn(pv[i]));
        // A layout: a0 (row g, keys 2t..), a1 (row g+8, keys 2t..), a2 (row g, keys 2t+8..), a3 (row g+8, ..)
        ph[0] = p_pack(hv[0], hv[1]);
        ph[1] = p_pack(hv[2], hv[3]);
        ph[2] = p_pack(hv[4], hv[5]);
        ph[3] = p_pack(hv[6], hv[7]);
        pl[0] = p_pack(pv[0] - hv[0], pv[1] - hv[1]);
        pl[1] = p_pack(pv[2] - hv[2], pv[3] - hv[3]);
        pl[2] = p_pack(pv[4] - hv[4], pv[5] - hv[5]);
        pl[3] = p_pack(pv[6] - hv[6], pv[7] - hv[7]);
#pragma unroll
        for (int nd = 0; nd < 8; ++nd) {  // dims [16nd, 16nd + 16): two n8 tiles
          const int key = 16 * ks + ((mi & 1) << 3) + mr, ch = 2 * nd + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          p_ldsm_x4_t(vt + sw_off(key, ch), b0, b1, b2, b3);
          p_mma(o[2 * nd], ph, b0, b1);
          p_mma(o[2 * nd], pl, b0, b1);
          p_mma(o[2 * nd + 1], ph, b2, b3);
          p_mma(o[2 * nd + 1], pl, b2, b3);
        }
      }
    }
    __syncthreads();  // the buffer is refilled next iteration
  }

  // ---- normalise and write rows gq and gq + 8 of this warp
  const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
  const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
  const int ra = wr + gq, rb = wr + gq + 8;
  bf16* out = reinterpret_cast<bf16*>(a.out);
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int d = 8 * n + 2 * tq;
    if (ra < nrows) {
      __nv_bfloat162 v = __floats2bfloat162_rn(o[n][0] * inv0, o[n][1] * inv0);
      *reinterpret_cast<__nv_bfloat162*>(out + (size_t)(r0 + ra) * a.out_row_stride + (size_t)h * kPHD + d) = v;
    }
    if (rb < nrows) {
      __nv_bfloat162 v = __floats2bfloat162_rn(o[n][2] * inv1, o[n][3] * inv1);
      *reinterpret_cast<__nv_bfloat162*>(out + (size_t)(r0 + rb) * a.out_row_stride + (size_t)h * kPHD + d) = v;
    }
  }
}

bool attn_prefill_mma_supported(const AttnRows& a, int dtype) {
  return dtype == Q2_BF16 && a.hd == kPHD && !a.seq_is_row && a.lens == nullptr && a.row_step == 1 &&
         a.nkv > 0 && a.nh % a.nkv == 0 && a.rows >= 16 && a.base >= 1 &&
         (a.q_row_stride % 8) == 0 && (a.kv_tok_stride % 8) == 0 && (a.out_row_stride % 2) == 0;
}

q2_status launch_attn_prefill_mma(const AttnRows& a, cudaStream_t st, bool pdl) {
  const size_t smem = PSmem::kTotal;
  Q2_CUDA_TRY(cudaFuncSetAttribute(attn_prefill_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem));
  dim3 grid((a.rows + kPQ - 1) / kPQ, a.nh);
  Q2_LAUNCH(attn_prefill_mma_kernel, grid, dim3(kPThreads), smem, st, pdl, a);
  return Q2_OK;
}

}  // namespace q2
