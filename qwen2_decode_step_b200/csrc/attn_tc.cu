// attn_tc.cu -- causal GQA attention of a block of query rows of one sequence
// (prefill) on the sm_100a tensor cores: tcgen05.mma with the score and
// output accumulators in tensor memory, operands in 128-byte-swizzled shared
// memory, K/V tiles by TMA.
//
// Work: an item is 128 query rows of one query head over the key tiles they
// see (longest row blocks of each head first).  The items that fill whole
// waves of the SMs run one CTA each; when the last, partial wave would leave
// SMs idle, each of its items is cut instead into ts ranges of key tiles
// (all items' first ranges first, so CTAs running together read nearby
// keys), one CTA per range.  A range's CTA writes its partial result (O
// unnormalised in fp32, the running max m and sum l of each row) to a slot,
// counts itself done on the item's counter, and the range that completes the
// count merges the item's ranges (O = sum 2^(m_k - M) O_k / sum 2^(m_k - M)
// l_k, M = max m_k) into the bf16 rows and resets the counter.  The usual
// write / fence / atomic pattern: no CTA waits for another.
// One CTA per item or range; 384 threads:
//   warp 0     TMA: the Q block once (two 64-dim boxes), then K and V tiles
//              of 128 keys into a three-stage ring
//   warp 1     allocates tensor memory; one thread issues the MMAs:
//                S_j  = Q K_j^T   M = 128 rows, N = 128 keys, K = 128 dims,
//                                 into TMEM S[j % 2] (fp32)
//                O   += P_j V_j   M = 128 rows, N = 128 dims, K = 128 keys,
//                                 into TMEM O (fp32), once with P's bf16 high
//                                 part and once with its low part (P keeps
//                                 16 significant bits); P is the A operand
//                                 in tensor memory, written over S_j's
//                                 columns; V is the MN-major operand (dims
//                                 contiguous, as the cache stores it)
//              in the order S_0, S_1, O += P_0 V_0, S_2, O += P_1 V_1, ...,
//              so a tile's scores are computed while the softmax of the tile
//              before runs
//   warps 4-11 softmax: two warps per 32 query rows (TMEM lanes), one per half
//              of the 128 key columns (and of the 128 output dims).  Each
//              reads its half of the row of S_j, applies the scale and the
//              causal mask, exchanges the partial row max with its partner,
//              keeps the running max m and its half of the sum l (O is
//              rescaled only when the max grows by more than 2^8, so most
//              tiles leave O untouched), writes P_j = 2^(s - m) as its bf16
//              truncation hi and bf16(P - hi) into tensor memory over its
//              half of S_j as the A operands of the P V products, and at the
//              end writes its half of O / l in bf16 (a key range: O, m and l
//              to the range's slot, then the counter and perhaps the merge).
// Every wait is bounded by a deadline; one that runs out sets value 2 in the
// caller's error word and the kernel carries on to its end.
//
// Definition followed: the attention of the Day-0 adaptation tutorial (step
// 5): scores q k^T * scale, causal mask (query i of a block at positions
// pos0.. sees keys j <= pos0 + i), stable softmax, times V; query head h reads
// kv head h / (nh / nkv).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kQB = 128;   // query rows per CTA (MMA M)
constexpr int kKB = 128;   // keys per tile
constexpr int kHD = 128;   // head dim
constexpr int kThreads = 384;   // warp 0 TMA, warp 1 MMA, warps 4-11 softmax
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;  // O is rescaled when the running max grows by more than this (log2)
constexpr uint64_t kDeadlineNs = 2000ull * 1000 * 1000;

constexpr size_t kBox = (size_t)128 * 64 * 2;  // one 128-row x 64-column bf16 box: 16 KB
constexpr size_t kQOff = 0;                    // Q: 2 boxes
constexpr size_t kKVOff = 2 * kBox;            // [kStages][K: 2 boxes | V: 2 boxes]
constexpr size_t kStage = 4 * kBox;
constexpr int kStages = 3;                      // K/V ring depth
constexpr size_t kBarOff = kKVOff + kStages * kStage;
constexpr size_t kSmem = kBarOff + 16 * 8 + 16 + 1024;  // barriers, TMEM base, alignment slack

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (gtimer() - t0 > kDeadlineNs) return false;
  }
}

// Shared-memory descriptor of a K-major, 128-byte-swizzled operand tile whose
// 8-row groups are 1024 bytes apart (a TMA box of 64 bf16 columns with
// 128-byte swizzle): start >> 4, leading offset 16 B (unused), stride offset
// 1024 B, descriptor version 1, swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
  return ((uint64_t)((saddr >> 4) & 0x3FFFu)) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

// Descriptor of an MN-major, 128-byte-swizzled operand: the MN dimension
// contiguous (64 elements = one 128-byte row of a swizzle atom), the K
// dimension along the rows (8 rows = one 1024-byte atom).  Leading offset:
// bytes between 64-element MN blocks (the next TMA box); stride offset: bytes
// between 8-row K groups (1024).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, uint32_t mn_block_bytes) {
  return ((uint64_t)((saddr >> 4) & 0x3FFFu)) | ((uint64_t)((mn_block_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, A K-major,
// B K-major (b_mn = 0) or MN-major (b_mn = 1), N = n, M = 128.
__host__ __device__ constexpr uint32_t idesc(int n, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(kQB >> 4) << 24);
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

// The same with A read from tensor memory (K-major: lane = row, two bf16 of
// consecutive k per 32-bit column).
__device__ __forceinline__ void mma_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (no wait).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
      "%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32: relative error
// near 2^-22, results below 2^-126 flushed to zero, 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct AttnTc {
  int rows;        // query rows of the chunk
  int nh, nkv;     // heads
  int pos0;        // position of query row 0 (row i sees keys 0 .. pos0 + i)
  int kv_x_step;   // K/V tensor maps: the tile origin of kv head g is at
  int kv_y_step;   // (x, y) = (g * kv_x_step, g * kv_y_step + first key)
  float scale;
  void* out;
  long long out_row_stride;  // elements
  int* err;
  int ntq;       // row blocks; item i is row block ntq - 1 - i % ntq of head i / ntq
  int n_whole;   // items 0 .. n_whole - 1 run whole, one CTA each
  int ts;        // the later items' key ranges (CTA n_whole + p: range p / n_tail of item n_whole + p % n_tail)
  float* part;   // [n_tail * ts] slots of kSlotFloats
  int* cnt;      // [n_tail] ranges done (0 between launches)
};

// A slot: O (fp32, [row][dim]), then m and l of each row.
constexpr int kSlotFloats = kQB * kHD + 2 * kQB;

// Key tiles of row block qt: up to the block's last visible key.
__host__ __device__ __forceinline__ int item_tiles(int rows, int pos0, int qt) {
  const int last_row = (qt * kQB + kQB < rows ? qt * kQB + kQB : rows) - 1;
  return (pos0 + last_row) / kKB + 1;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnTc a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [kStages]
  uint64_t* kv_empty = bars + 4;  // [kStages]
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;    // [2]
  uint64_t* o_done = bars + 11;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(bars + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.ntq * a.nh, n_tail = n_items - a.n_whole;
  const int piece = (int)blockIdx.x - a.n_whole;  // >= 0: a key range of a tail item
  const int item = piece < 0 ? (int)blockIdx.x : a.n_whole + piece % n_tail;
  const int qt = a.ntq - 1 - item % a.ntq;  // the longest (last) row blocks of a head first
  const int h = item / a.ntq, kvh = h / (a.nh / a.nkv);
  const int q0 = qt * kQB;
  const int nkt = item_tiles(a.rows, a.pos0, qt);  // key tiles up to the block's last visible key
  const int jb = piece < 0 ? 0 : (piece / n_tail) * nkt / a.ts;           // this CTA's key tiles:
  const int n = (piece < 0 ? nkt : (piece / n_tail + 1) * nkt / a.ts) - jb;  // jb .. jb + n - 1
  const int keys_end = a.pos0 + a.rows;  // keys written so far (later rows are stale)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
    }
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {  // S[0], S[1], O: 3 x 128 fp32 columns (allocated as 512)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_base_s)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_base_s);
  const uint32_t tS0 = tmem, tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * kBox);
      for (int b = 0; b < 2; ++b) tma_load_2d(smem + kQOff + b * kBox, &tq, h * kHD + 64 * b, q0, q_full);
      const int xbase = kvh * a.kv_x_step, ybase = kvh * a.kv_y_step;
      for (int j = 0; j < n; ++j) {  // the CTA's j-th tile: key tile jb + j
        const int kv = j % kStages;
        if (j >= kStages && !wait_bar(&kv_empty[kv], (uint32_t)((j / kStages - 1) & 1))) atomicOr(a.err, 2);
        uint8_t* st = smem + kKVOff + kv * kStage;
        mbar_arrive_expect_tx(&kv_full[kv], 4 * kBox);
        for (int b = 0; b < 2; ++b) {
          tma_load_2d(st + b * kBox, &tk, xbase + 64 * b, ybase + (jb + j) * kKB, &kv_full[kv]);
          tma_load_2d(st + (2 + b) * kBox, &tv, xbase + 64 * b, ybase + (jb + j) * kKB, &kv_full[kv]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t id_s = idesc(kKB, 0);  // S = Q K^T: both K-major (dims contiguous)
      constexpr uint32_t id_o = idesc(kHD, 1);  // O += P V: P K-major (keys contiguous), V MN-major
      const uint32_t qa = smem_u32(smem + kQOff);
      if (!wait_bar(q_full, 0)) atomicOr(a.err, 2);
      auto pv = [&](int j) {  // O += P_j V_j, P_j in the columns of S[j % 2]
        const int s = j & 1, kv = j % kStages;
        if (!wait_bar(&p_full[s], (uint32_t)((j >> 1) & 1))) atomicOr(a.err, 2);
        fence_after();
        const uint32_t tp = tS0 + (uint32_t)(s * kKB);
        const uint32_t va = smem_u32(smem + kKVOff + (size_t)kv * kStage + 2 * kBox);
#pragma unroll
        for (int k = 0; k < kKB / 16; ++k) {  // 16 keys per MMA
          // keys 64 hf + 16 kk ..: high part at column 64 hf + 8 kk, low part 32 further
          const uint32_t pc = (uint32_t)(64 * (k >> 2) + 8 * (k & 3));
          const uint64_t db = desc_mnmajor(va + (uint32_t)(k * 16 * 128), (uint32_t)kBox);
          mma_ta(tO, tp + pc, db, id_o, (j > 0 || k > 0) ? 1u : 0u);
          mma_ta(tO, tp + pc + 32, db, id_o, 1u);
        }
        commit(o_done);
        commit(&kv_empty[kv]);
      };
      for (int j = 0; j < n; ++j) {
        const int s = j & 1, kv = j % kStages;
        if (!wait_bar(&kv_full[kv], (uint32_t)((j / kStages) & 1))) atomicOr(a.err, 2);
        fence_after();
        const uint32_t ka = smem_u32(smem + kKVOff + (size_t)kv * kStage);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k) {  // 16 dims per MMA
          const uint32_t off = (uint32_t)((k >> 2) * kBox) + (uint32_t)((k & 3) * 32);
          mma(tS0 + (uint32_t)(s * kKB), desc_kmajor(qa + off), desc_kmajor(ka + off), id_s, k > 0 ? 1u : 0u);
        }
        commit(&s_full[s]);
        if (j > 0) pv(j - 1);
      }
      if (n > 0) pv(n - 1);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    // Two warps per group of 32 rows (TMEM lanes): warps 4-7 take key columns
    // 0-63 of their rows (and output dims 0-63), warps 8-11 columns 64-127.
    // Thread r owns query row r.  The pair exchanges its partial row maxima
    // each tile through the first 1 KB of the tile's K buffer, which S has
    // been computed from and which is not refilled before P is published.
    const int sw = warp - 4;                 // 0..7
    const int rg = sw & 3, half = sw >> 2;   // lane quarter, column half
    const int r = rg * 32 + lane;            // query row of the block = TMEM lane
    const int cb = 64 * half;                // this warp's first column
    const uint32_t lane_off = (uint32_t)(rg * 32) << 16;
    const int qpos = a.pos0 + q0 + r;        // this row sees keys 0 .. qpos
    const float sl2 = a.scale * kLog2e;
    // the two warps of a row group meet on their own named barrier (1 + rg, 64 threads)
    auto pair_sync = [rg] { asm volatile("bar.sync %0, 64;" ::"r"(1 + rg) : "memory"); };
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1, kv = j % kStages;
      if (!wait_bar(&s_full[s], (uint32_t)((j >> 1) & 1))) atomicOr(a.err, 2);
      fence_after();
      // This warp's half of the row's raw scores, kept in registers for both
      // passes; keys beyond the row's position become -inf (only on the
      // tiles the block's diagonal crosses), so 2^(s - m) is 0 there.  The
      // max is taken over the raw scores as a tree and scaled once: scaling
      // by a positive factor and rounding both keep the order.
      const int kb = (jb + j) * kKB;
      const bool visible = kb + kKB - 1 <= a.pos0 + q0;  // every row of the block sees the whole tile
      uint32_t sv[64];
      tmem_ld32_nowait(tS0 + lane_off + (uint32_t)(s * kKB + cb), sv);
      tmem_ld32_nowait(tS0 + lane_off + (uint32_t)(s * kKB + cb + 32), sv + 32);
      tmem_ld_wait();
      if (!visible) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (kb + cb + e > qpos) sv[e] = __float_as_uint(-INFINITY);
      }
      float mh;
      {
        float t[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) t[e] = fmaxf(__uint_as_float(sv[e]), __uint_as_float(sv[e + 32]));
#pragma unroll
        for (int w = 16; w > 0; w >>= 1)
#pragma unroll
          for (int e = 0; e < w; ++e) t[e] = fmaxf(t[e], t[e + w]);
        mh = t[0];
      }
      if (mh != -INFINITY) mh *= sl2;
      // the row's max: this half's and the partner's (the K buffer's TMA
      // writes are complete: kv_full's phase is done)
      if (!wait_bar(&kv_full[kv], (uint32_t)((j / kStages) & 1))) atomicOr(a.err, 2);
      float* xch = reinterpret_cast<float*>(smem + kKVOff + (size_t)kv * kStage);
      xch[half * kQB + r] = mh;
      pair_sync();
      const float mt = fmaxf(mh, xch[(half ^ 1) * kQB + r]);
      // This row's max moves when the tile's max exceeds it by more than 2^8
      // (or on the first tile); O and l are then rescaled.  tcgen05.ld / st are
      // warp-collective, so the warp rescales when any of its rows needs it,
      // the other rows by 1.  Both warps of a row take the same decision.
      float alpha = 1.f;
      if (mt > m_run + kRescale || m_run == -INFINITY) {
        const float mnew = fmaxf(mt, m_run);
        if (m_run != -INFINITY) alpha = exp2f(m_run - mnew);
        if (mnew != -INFINITY) m_run = mnew;
      }
      l_run *= alpha;
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O is rescaled once the product of the tile before is done
        if (!wait_bar(o_done, (uint32_t)((j - 1) & 1))) atomicOr(a.err, 2);
        fence_after();
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t ov[32];
          tmem_ld32_nowait(tO + lane_off + (uint32_t)(cb + 32 * c), ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(tO + lane_off + (uint32_t)(cb + 32 * c), ov);
        }
        tmem_st_wait();
      }
      // P = 2^(s - m) of this half's 64 keys as bf16 high and low parts,
      // written over this half's 64 columns of S: the high parts of keys
      // 2 e, 2 e + 1 in column e, the low parts 32 columns further.  The high
      // part is P's top 16 bits (P truncated to bf16), the low part P - high
      // (exact in fp32, below 2^-7 P) rounded to bf16, so high + low is P to
      // within 2^-16 of it.  S[j % 2] is not read again, and P_j is read by
      // the P V product before S_(j+2) is written there.
      // (key pairs on the packed two-lane fp32 FMA and add: the same
      // roundings as two scalar operations)
      const float nm = m_run == -INFINITY ? 0.f : -m_run;
      const float2 sl2x2 = make_float2(sl2, sl2), nmx2 = make_float2(nm, nm);
      float2 ls = make_float2(0.f, 0.f);
      uint32_t phi[32], plo[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sl2x2, nmx2);
        const float2 pp = make_float2(ex2(x.x), ex2(x.y));
        ls = __fadd2_rn(ls, pp);
        const uint32_t b0 = __float_as_uint(pp.x), b1 = __float_as_uint(pp.y);
        phi[e] = __byte_perm(b0, b1, 0x7632);  // the upper halves: key 2 e low, key 2 e + 1 high
        // minus the high parts: the top 16 bits with the sign flipped
        const float2 lo = __fadd2_rn(pp, make_float2(__uint_as_float((b0 & 0xFFFF0000u) ^ 0x80000000u),
                                                      __uint_as_float((b1 & 0xFFFF0000u) ^ 0x80000000u)));
        const __nv_bfloat162 l2 = __float22bfloat162_rn(lo);
        plo[e] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      const float lsum = ls.x + ls.y;
      tmem_st32(tS0 + lane_off + (uint32_t)(s * kKB + cb), phi);
      tmem_st32(tS0 + lane_off + (uint32_t)(s * kKB + cb + 32), plo);
      tmem_st_wait();
      l_run += lsum;
      // keys past the ones written so far are stale cache rows (possibly not
      // finite, and 0 * inf would poison the sum): zero them in V
      if (jb + j == nkt - 1 && kb + kKB > keys_end) {
        uint8_t* vt = smem + kKVOff + (size_t)kv * kStage + 2 * kBox;
        const int row0 = keys_end - kb;  // first stale row of the tile
        for (int i = sw * 32 + lane; i < (kKB - row0) * 16; i += 256) {  // 16 chunks of 16 bytes per row
          const int vr = row0 + i / 16, ch = i % 16;
          *reinterpret_cast<uint4*>(vt + (ch >> 3) * kBox + vr * 128 + (((ch & 7) ^ (vr & 7)) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();  // the exchange and zeroed V rows: the async proxy refills or reads them next
      fence_before();
      mbar_arrive(&p_full[s]);
    }
    // ---- the last product, then O / l in bf16 (or O, m, l to the range's
    // slot): the two halves' sums are added through the Q buffer (free once
    // every product is done)
    if (n > 0 && !wait_bar(o_done, (uint32_t)((n - 1) & 1))) atomicOr(a.err, 2);
    fence_after();
    float* lx = reinterpret_cast<float*>(smem + kQOff);
    lx[half * kQB + r] = l_run;
    pair_sync();
    const float lr = lx[r] + lx[kQB + r];
    const int row = q0 + r;
    bf16* out = reinterpret_cast<bf16*>(a.out) + (size_t)row * a.out_row_stride + (size_t)h * kHD + cb;
    if (piece < 0) {
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t ov[32];
        tmem_ld32_nowait(tO + lane_off + (uint32_t)(cb + 32 * c), ov);
        tmem_ld_wait();
        if (row < a.rows) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float f[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) f[t] = __uint_as_float(ov[e + t]) * inv;
            *reinterpret_cast<uint4*>(out + 32 * c + e) = pack16<bf16>(f);
          }
        }
      }
    } else {
      const int t = item - a.n_whole;
      float* sl = a.part + (size_t)piece * kSlotFloats;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t ov[32];
        tmem_ld32_nowait(tO + lane_off + (uint32_t)(cb + 32 * c), ov);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(sl + (size_t)r * kHD + cb + 32 * c);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                               __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
      }
      sl[kQB * kHD + half * kQB + r] = half == 0 ? m_run : lr;
      // count the range done; the one that completes the count merges
      __threadfence();
      int* last = reinterpret_cast<int*>(lx + 2 * kQB);
      asm volatile("bar.sync 5, 256;" ::: "memory");
      if (sw == 0 && lane == 0) {
        const int done = atomicAdd(&a.cnt[t], 1);
        if (done == a.ts - 1) a.cnt[t] = 0;  // every range has counted: ready for the next launch
        *last = done == a.ts - 1;
      }
      asm volatile("bar.sync 5, 256;" ::: "memory");
      if (*last) {
        __threadfence();
        float mm = -INFINITY;
        for (int k = 0; k < a.ts; ++k)
          mm = fmaxf(mm, __ldcg(a.part + (size_t)(k * n_tail + t) * kSlotFloats + kQB * kHD + r));
        float o[64], ll = 0.f;
#pragma unroll
        for (int d = 0; d < 64; ++d) o[d] = 0.f;
        for (int k = 0; k < a.ts; ++k) {
          const float* sk = a.part + (size_t)(k * n_tail + t) * kSlotFloats;
          const float mk = __ldcg(sk + kQB * kHD + r);
          if (mk == -INFINITY) continue;  // the row sees no key in this range
          const float w = exp2f(mk - mm);
          ll += w * __ldcg(sk + kQB * kHD + kQB + r);
          const float4* src = reinterpret_cast<const float4*>(sk + (size_t)r * kHD + cb);
#pragma unroll
          for (int d = 0; d < 16; ++d) {
            const float4 v = __ldcg(src + d);
            o[4 * d] += w * v.x;
            o[4 * d + 1] += w * v.y;
            o[4 * d + 2] += w * v.z;
            o[4 * d + 3] += w * v.w;
          }
        }
        const float inv = ll > 0.f ? 1.f / ll : 0.f;
        if (row < a.rows) {
#pragma unroll
          for (int e = 0; e < 64; e += 8) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = o[e + u] * inv;
            *reinterpret_cast<uint4*>(out + e) = pack16<bf16>(f);
          }
        }
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
  }
}

// K/V either head-major (positions of one kv head contiguous, the cache's
// layout: [nkv][positions][hd]) or token-major (the heads of one position
// contiguous: [positions][nkv][hd]).
static bool kv_head_major(const AttnRows& a) { return a.kv_tok_stride == kHD && a.kv_head_stride % kHD == 0; }
static bool kv_token_major(const AttnRows& a) {
  return a.kv_head_stride == kHD && a.kv_tok_stride % 8 == 0 && a.kv_tok_stride >= (long long)a.nkv * kHD;
}

// K and V of the rows' sequence (a.fixed_seq)
static const bf16* seq_k(const AttnRows& a) {
  return reinterpret_cast<const bf16*>(a.k) + (size_t)a.fixed_seq * a.kv_seq_stride;
}
static const bf16* seq_v(const AttnRows& a) {
  return reinterpret_cast<const bf16*>(a.v) + (size_t)a.fixed_seq * a.kv_seq_stride;
}

// The work-split scratch: the tail items' counters, then their ranges' slots.
constexpr int kMaxTs = 6;
constexpr size_t kCntBytes = 4096;
size_t attn_tc_ws_bytes() { return kCntBytes + (size_t)num_sms() * kMaxTs * kSlotFloats * sizeof(float); }

int attn_tc_slot_capacity(int sms) { return sms * kMaxTs; }
int attn_tc_counter_capacity() { return (int)(kCntBytes / sizeof(int)); }

// The items that fill whole waves run whole; the last wave's items are cut
// into ts key ranges when that shortens it: with n_tail items left of average
// length len tiles, the tail takes about ceil(n_tail ts / SMs) (len / ts + c)
// tile times, c ~ 3 tiles for a CTA's start, pipeline fill and partial write;
// a ts is taken only if it saves 3 %.  ts is at most kMaxTs and the shortest
// tail item's tile count (every range has a tile); n_tail < SMs, so the
// ranges fit SMs x kMaxTs slots.
void attn_tc_plan(int rows, int pos0, int nh, int sms, bool split_ok, int* n_whole, int* ts) {
  const int ntq = (rows + kQB - 1) / kQB, items = ntq * nh;
  *n_whole = items;
  *ts = 1;
  const int n_tail = items % sms;
  if (!split_ok || n_tail == 0) return;
  long long sum = 0;
  int shortest = 1 << 30;
  for (int i = items - n_tail; i < items; ++i) {
    const int nt = item_tiles(rows, pos0, ntq - 1 - i % ntq);
    sum += nt;
    shortest = std::min(shortest, nt);
  }
  const double len = (double)sum / n_tail, c = 3.0;
  double best = len + c;
  for (int t = 2; t <= std::min(kMaxTs, shortest); ++t) {
    const double cost = (double)((n_tail * t + sms - 1) / sms) * (len / t + c);
    if (cost < 0.97 * best) {
      best = cost;
      *ts = t;
    }
  }
  if (*ts > 1) *n_whole = items - n_tail;
}

bool attn_tc_supported(const AttnRows& a, int dtype) {
  return dtype == Q2_BF16 && a.hd == kHD && !a.seq_is_row && a.lens == nullptr && a.row_step == 1 &&
         a.nkv > 0 && a.nh % a.nkv == 0 && a.rows >= 16 && a.base >= 1 && a.fixed_seq >= 0 &&
         (a.q_row_stride % 8) == 0 && (kv_head_major(a) || kv_token_major(a)) && (a.out_row_stride % 8) == 0 &&
         (reinterpret_cast<uintptr_t>(a.q) & 15) == 0 && (reinterpret_cast<uintptr_t>(seq_k(a)) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(seq_v(a)) & 15) == 0 && (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
}

q2_status launch_attn_tc(const AttnRows& a, void* ws, int* err, cudaStream_t st) {
  if (a.rows == 0) return Q2_OK;
  const int pos0 = a.base - 1;
  const long long keys = (long long)pos0 + a.rows;  // keys visible to the last row
  CUtensorMap tq, tk, tv;
  // Q as [rows, nh * hd]
  Q2_TRY(make_tmap_2d_bf16(&tq, a.q, (uint64_t)a.rows, (uint64_t)a.nh * kHD, (uint64_t)a.q_row_stride * 2, kQB,
                           64, 128));
  AttnTc p;
  if (kv_head_major(a)) {
    // [nkv * positions, hd]: kv head g starts at row g * positions
    const long long kv_rows = a.kv_head_stride / kHD;
    Q2_TRY(make_tmap_2d_bf16(&tk, seq_k(a), (uint64_t)a.nkv * kv_rows, kHD, kHD * 2, kKB, 64, 128));
    Q2_TRY(make_tmap_2d_bf16(&tv, seq_v(a), (uint64_t)a.nkv * kv_rows, kHD, kHD * 2, kKB, 64, 128));
    p.kv_x_step = 0;
    p.kv_y_step = (int)kv_rows;
  } else {
    // [positions, nkv * hd]: kv head g starts at column g * hd; no row past
    // the visible keys exists in the map (it reads as zeros)
    Q2_TRY(make_tmap_2d_bf16(&tk, seq_k(a), (uint64_t)keys, (uint64_t)a.nkv * kHD, (uint64_t)a.kv_tok_stride * 2,
                             kKB, 64, 128));
    Q2_TRY(make_tmap_2d_bf16(&tv, seq_v(a), (uint64_t)keys, (uint64_t)a.nkv * kHD, (uint64_t)a.kv_tok_stride * 2,
                             kKB, 64, 128));
    p.kv_x_step = kHD;
    p.kv_y_step = 0;
  }
  p.rows = a.rows;
  p.nh = a.nh;
  p.nkv = a.nkv;
  p.pos0 = pos0;
  p.scale = a.scale;
  p.out = a.out;
  p.out_row_stride = a.out_row_stride;
  p.err = err;
  p.ntq = (a.rows + kQB - 1) / kQB;
  const int items = p.ntq * a.nh;
  attn_tc_plan(a.rows, pos0, a.nh, num_sms(), ws != nullptr, &p.n_whole, &p.ts);
  p.cnt = reinterpret_cast<int*>(ws);
  p.part = ws ? reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kCntBytes) : nullptr;
  Q2_CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
  const int grid = p.n_whole + (items - p.n_whole) * p.ts;
  Q2_LAUNCH(attn_tc_kernel, dim3(grid), dim3(kThreads), kSmem, st, false, tq, tk, tv, p);
  return Q2_OK;
}

}  // namespace q2
