// pdecode.cu -- the persistent bf16 decode step (see pdecode.h).
//
// Numerics are those of the operator-by-operator path: each operator's
// output is rounded to bf16 where the operator would write it back.
#include <limits.h>

#include "common.cuh"
#include "pdecode.h"
#include "tma.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kC = kPConsumers;             // consumer warps
constexpr int kThreads = (kC + 2) * 32;     // + the producer and the epilogue warp
constexpr int kSlot = 8 * (1536 * 2 + 64);  // ring slot: 8 padded rows of K = 1536
constexpr int kRowPad = 64;                 // bytes between staged rows beyond K (bank spread)
constexpr int kActPad = 32;                 // bf16 elements of padding per activation row
constexpr int kEpiRows = 64;                // output rows per CTA with staged epilogue operands
constexpr int kAT = 64;                     // attention keys per tile
constexpr int kHD = 128;                    // head dim of this kernel
constexpr int kTileBytes = kAT * kHD * 2;   // one K (or V) tile
constexpr int kAGMax = 8;                   // query heads per kv head
constexpr int kNHMax = 16;                  // query heads
constexpr int kSplitMax = 64;
constexpr size_t kSmemMax = 232448;         // 227 KB per CTA
constexpr uint64_t kDeadlineNs = 200ull * 1000 * 1000;  // 200 ms
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory map (offsets from a 1024-byte aligned base).
struct PGeo {
  int ring;          // weight ring slots
  int act_elems;     // per-token activation capacity (max of H, I, qd)
  size_t o_ring, o_act, o_qs, o_S, o_ml, o_red, o_bars, o_flag, o_acc, o_epi, total;
};

__host__ __device__ inline size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

PGeo make_geo(int mt, int act_elems) {
  PGeo g;
  g.act_elems = act_elems;
  for (int ring = 8; ring >= 1; --ring) {
    size_t o = 2 * 2 * (size_t)kTileBytes;  // attention K/V tiles, two stages
    g.o_ring = o;
    o += (size_t)ring * kSlot;
    g.o_act = o;
    o = up(o + (size_t)mt * (act_elems + kActPad) * 2, 16);
    g.o_qs = o;
    o += kAGMax * kHD * 4;
    g.o_S = o;
    o += kAGMax * kAT * 4;
    g.o_ml = o;
    o += 3 * kAGMax * 4;
    g.o_red = o;
    o += kC * 4 * 4;
    g.o_bars = up(o, 8);
    // full[ring], empty[ring], posted[ring + 1], epid[ring + 1], abar[2]
    o = g.o_bars + (2 * (size_t)ring + 2 * (size_t)(ring + 1) + 2) * 8;
    o = up(o, 8);
    g.o_flag = o;
    o += 16;
    g.o_acc = o;  // per-warp row-group sums [ring + 1][kC][8 rows][4 tokens]
    o += (size_t)(ring + 1) * kC * 8 * 4 * 4;
    g.o_epi = o;  // staged epilogue operands: bias, RoPE cos/sin, residual rows
    o += (size_t)kEpiRows * 4 * (1 + 2 + 4);
    g.ring = ring;
    g.total = o + 1024;  // slack for aligning the base
    if (g.total <= kSmemMax) break;
  }
  return g;
}

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// try_wait that lets the hardware suspend the thread for up to `ns` while the
// phase is still open (a waiting warp then takes no issue slots).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// mbarrier wait with a deadline; false if it ran out.
__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (;;) {
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (gtimer() - t0 > kDeadlineNs) return false;
  }
}

__device__ __forceinline__ unsigned atom_add_release(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void csync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kC * 32) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ float silu_mul(float gv, float uv) { return uv * (gv / (1.0f + expf(-gv))); }

// c += A . B for one m16n8k16 tile, bf16 operands, fp32 accumulators.  A rows
// 8..15 are zero: only a0 (row g, k pair 2t) and a2 (row g, k pair 2t + 8) are
// passed; b0 and b1 are column g's k pairs 2t and 2t + 8.
__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a2, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ int swz(int r, int c) {
  return r * 128 + ((((c >> 3) ^ (r & 7)) << 4) | ((c & 7) << 1));
}

enum { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_GU = 3, PH_DOWN = 4, PH_HEAD = 5 };

// A weight phase streams W [N][K] in stages of R rows x KT columns (kb = K / KT
// column blocks per group of R rows); each CTA owns the row groups [gb, ge).
struct WPhase {
  const bf16* w;
  int N, K, R, KT, kb, stride, kind, gb, ge;
};

// Rows per group: 8, or 4 where that cuts the rows of the busiest CTA by at
// least an eighth (small N, e.g. the o and down projections).
__host__ __device__ inline int phase_rows(int N, int G) {
  const int c8 = (N + 8 * G - 1) / (8 * G) * 8, c4 = (N + 4 * G - 1) / (4 * G) * 4;
  return 8 * c4 <= 7 * c8 ? 4 : 8;
}

// Column blocks: the fewest with KT a multiple of 256 whose R padded rows fit a slot.
__host__ __device__ inline int phase_kblocks(int K, int R) {
  if (K % 256 != 0) return 0;
  for (int kb = 1; kb <= K / 256; ++kb)
    if ((K / 256) % kb == 0 && (size_t)R * ((size_t)(K / kb) * 2 + kRowPad) <= (size_t)kSlot) return kb;
  return 0;
}

__device__ __forceinline__ int phase_kind(const PDecode& p, int ph) {
  return ph == 5 * p.L ? PH_HEAD : ph % 5;
}

__device__ __forceinline__ bool weight_phase(const PDecode& p, int ph, int bid, int G, WPhase& wp) {
  const int kind = phase_kind(p, ph);
  if (kind == PH_ATTN) return false;
  const PLayer* Lw = kind == PH_HEAD ? nullptr : &p.layers[ph / 5];
  switch (kind) {
    case PH_QKV: wp.w = (const bf16*)Lw->wqkv; wp.N = p.qkvd; wp.K = p.H; break;
    case PH_O: wp.w = (const bf16*)Lw->wo; wp.N = p.H; wp.K = p.qd; break;
    case PH_GU: wp.w = (const bf16*)Lw->wgu; wp.N = 2 * p.I; wp.K = p.H; break;
    case PH_DOWN: wp.w = (const bf16*)Lw->wd; wp.N = p.H; wp.K = p.I; break;
    default: wp.w = (const bf16*)p.lm_head; wp.N = p.V; wp.K = p.H; break;
  }
  wp.R = phase_rows(wp.N, G);
  wp.kb = phase_kblocks(wp.K, wp.R);
  wp.KT = wp.K / wp.kb;
  wp.stride = wp.KT * 2 + kRowPad;
  wp.kind = kind;
  const int ng = (wp.N + wp.R - 1) / wp.R;
  wp.gb = (int)((long long)bid * ng / G);
  wp.ge = (int)((long long)(bid + 1) * ng / G);
  return true;
}

// The sequence of weight stages one CTA streams: phase by phase, for each of
// its row groups the kb column blocks in order (no divisions per stage).
struct StageIter {
  WPhase wp;
  int ph, grp, kblk;
  __device__ void enter(const PDecode& p, int bid, int G, int nph) {
    for (; ph < nph; ++ph) {
      if (!weight_phase(p, ph, bid, G, wp)) continue;
      grp = wp.gb;
      kblk = 0;
      if (wp.gb < wp.ge) return;
    }
    grp = 0;
    wp.ge = 0;
  }
  __device__ void begin(const PDecode& p, int bid, int G, int nph) {
    ph = 0;
    enter(p, bid, G, nph);
  }
  __device__ bool valid() const { return grp < wp.ge; }
  __device__ void next(const PDecode& p, int bid, int G, int nph) {
    if (++kblk < wp.kb) return;
    kblk = 0;
    if (++grp < wp.ge) return;
    ++ph;
    enter(p, bid, G, nph);
  }
  __device__ int rows() const { return min(wp.R, wp.N - grp * wp.R); }
  __device__ uint32_t bytes() const { return (uint32_t)rows() * wp.KT * 2; }
  // row r of the stage in global memory
  __device__ const bf16* src(int r) const {
    return wp.w + (size_t)(grp * wp.R + r) * wp.K + (size_t)kblk * wp.KT;
  }
};

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

}  // namespace

// ======================================================================
template <int MT>
__global__ void __launch_bounds__(kThreads, 1) pdecode_kernel(const PDecode p, const PGeo g,
                                                              const __grid_constant__ CUtensorMap kmap,
                                                              const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* tiles = smem;  // [2 stages][K | V] attention tiles (128B-swizzled boxes)
  uint8_t* ring = smem + g.o_ring;
  bf16* act = reinterpret_cast<bf16*>(smem + g.o_act);
  float* qs = reinterpret_cast<float*>(smem + g.o_qs);
  float* S = reinterpret_cast<float*>(smem + g.o_S);
  float* ms = reinterpret_cast<float*>(smem + g.o_ml);
  float* ls = ms + kAGMax;
  float* al = ls + kAGMax;
  float* red = reinterpret_cast<float*>(smem + g.o_red);
  // Weight ring: full[slot] completes when a stage's bytes have landed,
  // empty[slot] when all kC consumer warps have passed the stage.  Every
  // consumer warp passes every stage, in order, computing only its own units,
  // so no waiter is ever more than one phase away from the barrier it waits
  // on and every parity wait is unambiguous.
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + g.o_bars);
  uint64_t* empty = full + g.ring;
  // Row-group accumulators: posted[a] completes when all kC consumer warps
  // have written their partial sums of the group on accumulator a, epid[a]
  // when the epilogue warp has finished that group.
  uint64_t* posted = empty + g.ring;
  uint64_t* epid = posted + g.ring + 1;
  uint64_t* abar = epid + g.ring + 1;
  int* s_flags = reinterpret_cast<int*>(smem + g.o_flag);
  int& s_flag = s_flags[0];
  int& s_last_merge = s_flags[1];
  int& s_pre = s_flags[2];  // attention tiles of this CTA's first item already in flight
  float* acc_s = reinterpret_cast<float*>(smem + g.o_acc);        // [ring + 1][kC][8][4]
  float* e_bias = reinterpret_cast<float*>(smem + g.o_epi);       // [kEpiRows]
  float2* e_cs = reinterpret_cast<float2*>(e_bias + kEpiRows);    // [kEpiRows / 2][4]
  float* e_x = reinterpret_cast<float*>(e_cs + kEpiRows / 2 * 4);  // [kEpiRows][4]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, bid = blockIdx.x;
  const int nph = p.run_head ? 5 * p.L + 1 : 5 * p.L;
  const int RING = g.ring;

  if (tid == 0) {
    for (int i = 0; i < RING; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kC);
    }
    for (int i = 0; i <= RING; ++i) {
      mbar_init(&posted[i], kC);
      mbar_init(&epid[i], 1);
    }
    mbar_init(&abar[0], 1);
    mbar_init(&abar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // Row-group accumulators: the producer issues a group's first stage only
  // after the epilogue warp has read the group that last used its accumulator.
  const int NACC = RING + 1;
  const unsigned ARRIVALS = 2u * (unsigned)G;  // per phase: consumers and epilogue warp of every CTA

  // The last arrival of the last phase wraps up the step: the step's token
  // per sequence (argmax over the CTAs' partials) and the lengths.
  auto wrap_up = [&](int t) {  // t: thread index within the caller's group
    __threadfence();
    if (t < p.B) {
      if (p.run_head) {
        float bv = -INFINITY;
        long long bi = LLONG_MAX;
        for (int b = 0; b < G; ++b) {
          const float v = __ldcg(p.am_val + b * 4 + t);
          const long long i = __ldcg(reinterpret_cast<const long long*>(p.am_idx) + b * 4 + t);
          if (am_better(v, i, bv, bi)) {
            bv = v;
            bi = i;
          }
        }
        p.next[t] = bi;
      }
      p.lens[t] += 1;
    }
  };

  // ================================================================ producer
  // Lane 0 waits for a free slot and arms its barrier; lanes r < rows then
  // issue the copy of row r, and lane 31 pulls a later stage into L2.  Before
  // the first stage of a group it also waits until the epilogue warp is done
  // with the group that last used the group's accumulator.
  if (warp == kC) {
    const uint64_t pol = policy_evict_first();
    // `ahead` runs p.l2_ahead stages in front of the ring and pulls them into
    // L2 (a group's rows are contiguous in W: all of them when its first
    // column block comes up), so HBM keeps streaming while the ring is full
    // (during the grid barriers and the attention phase).
    StageIter cur, ahead;
    cur.begin(p, bid, G, nph);
    ahead.begin(p, bid, G, nph);
    auto prefetch = [&](const StageIter& a) {
      if (lane == 31 && a.kblk == 0) bulk_prefetch_l2(a.src(0), (uint32_t)a.rows() * a.wp.K * 2);
    };
    for (int i = 0; i < p.l2_ahead && ahead.valid(); ++i, ahead.next(p, bid, G, nph)) prefetch(ahead);
    int slot = 0;
    uint32_t par = 0;
    int acc_i = 0;          // accumulator of the next group
    long long groups = 0;   // groups started
    for (long long gs = 0; cur.valid(); ++gs, cur.next(p, bid, G, nph)) {
      if (lane == 0) {
        // Reuse of a slot waits until every consumer warp has passed its
        // previous use (their reads of the slot are complete by then).
        if (gs >= RING && !mwait(&empty[slot], par ^ 1u)) atomicOr(p.err, 2);
        if (cur.kblk == 0) {
          if (groups >= NACC && !mwait(&epid[acc_i], (uint32_t)((groups / NACC - 1) & 1)))
            atomicOr(p.err, 2);
          ++groups;
          acc_i = acc_i + 1 == NACC ? 0 : acc_i + 1;
        }
        mbar_arrive_expect_tx(&full[slot], cur.bytes());
      }
      __syncwarp();
      if (lane < cur.rows())  // one copy per row: rows land wp.stride bytes apart
        bulk_g2s_evict_first(ring + (size_t)slot * kSlot + (size_t)lane * cur.wp.stride, cur.src(lane),
                             (uint32_t)cur.wp.KT * 2, &full[slot], pol);
      if (ahead.valid()) {
        prefetch(ahead);
        ahead.next(p, bid, G, nph);
      }
      if (++slot == RING) {
        slot = 0;
        par ^= 1u;
      }
    }
    return;
  }

  // ========================================================= epilogue warp
  // Finishes every row group once its partial sums are posted (lane (r, m):
  // row r, token m), and signals each phase's end to the grid once that
  // phase's last group is written.
  if (warp == kC + 1) {
    StageIter epi;
    epi.begin(p, bid, G, nph);
    const int r = lane >> 2, m = lane & 3;
    float best_v = -INFINITY;  // lm_head argmax of token m over this lane's rows
    long long best_i = LLONG_MAX;
    int arrived = 0;  // phases [0, arrived) signalled
    auto signal_until = [&](int ph_end) {
      for (; arrived < ph_end; ++arrived) {
        if (phase_kind(p, arrived) == PH_HEAD) {  // this CTA's argmax partial per token
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
            const long long oi = __shfl_xor_sync(0xffffffffu, best_i, o);
            if (am_better(ov, oi, best_v, best_i)) {
              best_v = ov;
              best_i = oi;
            }
          }
          if (lane < 4) {
            p.am_val[bid * 4 + lane] = best_v;
            p.am_idx[bid * 4 + lane] = best_i;
          }
        }
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          if (p.trace) atomicMax(&p.trace[arrived * 4 + 0], (unsigned long long)gtimer());
          last = atom_add_release(&p.sync[arrived], 1u) == ARRIVALS - 1 && arrived == nph - 1;
        }
        if (__shfl_sync(0xffffffffu, last, 0)) wrap_up(lane);
      }
    };
    signal_until(epi.valid() ? epi.ph : nph);
    int acc_i = 0;
    long long groups = 0;
    for (; epi.valid(); epi.next(p, bid, G, nph), signal_until(epi.valid() ? epi.ph : nph)) {
      const WPhase& wp = epi.wp;
      if (epi.kblk != wp.kb - 1) continue;  // the group ends at its last column block
      const int ai = acc_i;
      acc_i = acc_i + 1 == NACC ? 0 : acc_i + 1;
      if (lane == 0 && !mwait(&posted[ai], (uint32_t)((groups / NACC) & 1))) atomicOr(p.err, 2);
      ++groups;
      __syncwarp();
      const float* acc = acc_s + ai * (kC * 32);
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kC; ++w) v += acc[w * 32 + r * 4 + m];
      const float vn = __shfl_down_sync(0xffffffffu, v, 4);  // row r + 1, token m
      __syncwarp();
      if (lane == 0) mbar_arrive(&epid[ai]);  // the accumulator is read
      const int R = wp.R, rows = epi.rows();
      const int n = epi.grp * R + r, i = n - wp.gb * R;  // output row, staged operand index
      if (r >= rows || m >= p.B) continue;
      const int kind = wp.kind, l = epi.ph / 5;
      if (kind == PH_O || kind == PH_DOWN) {
        const bf16 xn = from_f<bf16>(e_x[i * 4 + m] + round_st<bf16>(v));
        reinterpret_cast<bf16*>(p.x)[(size_t)m * p.H + n] = xn;
        e_x[i * 4 + m] = __bfloat162float(xn);
      } else if (kind == PH_GU) {
        if ((r & 1) == 0) {
          const float gv = round_st<bf16>(v), uv = round_st<bf16>(vn);
          reinterpret_cast<bf16*>(p.s)[(size_t)m * p.I + (n >> 1)] = from_f<bf16>(silu_mul(gv, uv));
        }
      } else if (kind == PH_QKV) {
        if ((r & 1) == 0) {
          const int hs = n / p.hd, j = (n % p.hd) >> 1, half = p.hd >> 1;
          const float va = round_st<bf16>(v + e_bias[i]);
          const float vb = round_st<bf16>(vn + e_bias[i + 1]);
          const size_t loff = (size_t)l * p.kv_layer_stride + (size_t)m * p.kv_seq_stride;
          const int pos = p.lens[m];
          if (hs < p.nh + p.nkv) {
            const float2 cs = e_cs[(i >> 1) * 4 + m];
            const bf16 ra = from_f<bf16>(va * cs.x - vb * cs.y);
            const bf16 rb = from_f<bf16>(vb * cs.x + va * cs.y);
            bf16* dst = hs < p.nh ? reinterpret_cast<bf16*>(p.qb) + (size_t)m * p.qd + (size_t)hs * p.hd
                                  : reinterpret_cast<bf16*>(p.kc) + loff +
                                        ((size_t)(hs - p.nh) * p.max_seq + pos) * p.hd;
            dst[j] = ra;
            dst[j + half] = rb;
          } else {
            bf16* vr = reinterpret_cast<bf16*>(p.vc) + loff +
                       ((size_t)(hs - p.nh - p.nkv) * p.max_seq + pos) * p.hd;
            vr[j] = from_f<bf16>(va);
            vr[j + half] = from_f<bf16>(vb);
          }
        }
      } else {  // PH_HEAD
        p.logits[(size_t)m * p.V + n] = v;
        if (am_better(v, n, best_v, best_i)) {
          best_v = v;
          best_i = n;
        }
      }
    }
    signal_until(nph);
    return;
  }

  // =============================================================== consumers
  const int ct = tid;
  const int G_q = p.nh / p.nkv;
  long long gs = 0;  // weight stages consumed so far (same sequence as the producer's)
  int r_slot = 0;    // ring slot and parity of the next stage
  uint32_t r_par = 0;
  int a_slot = 0;    // row-group accumulator of the next group
  int ac = 0;        // attention tile loads issued so far
  const bf16* X = reinterpret_cast<const bf16*>(p.x);
  // TMA load of K/V tile t of (layer l, sequence b, kv head gq) into
  // attention buffer stage li & 1 (issued by one thread).
  auto tile_issue = [&](int l, int b, int gq, int t, int li) {
    const int stg = li & 1;
    const int row_base = ((l * p.Bmax + b) * p.nkv + gq) * p.max_seq;
    uint8_t* kt = tiles + (size_t)stg * 2 * kTileBytes;
    uint8_t* vt = kt + kTileBytes;
    mbar_arrive_expect_tx(&abar[stg], 2 * kTileBytes);
#pragma unroll
    for (int bx = 0; bx < kHD / 64; ++bx) {
      tma_load_2d(kt + bx * 8192, &kmap, bx * 64, row_base + t * kAT, &abar[stg]);
      tma_load_2d(vt + bx * 8192, &vmap, bx * 64, row_base + t * kAT, &abar[stg]);
    }
  };
  // Work item `item` of an attention phase: sequence, kv head, split and tile range.
  struct AItem {
    int b, gq, split, L, ntiles, tps, t0, t1;
  };
  auto attn_geom = [&](int item) {
    AItem a;
    a.split = item / (p.B * p.nkv);
    const int rem = item % (p.B * p.nkv);
    a.b = rem / p.nkv;
    a.gq = rem % p.nkv;
    a.L = p.lens[a.b] + 1;
    a.ntiles = (a.L + kAT - 1) / kAT;
    const int active = min(p.nsplit, a.ntiles);
    a.tps = (a.ntiles + active - 1) / active;
    a.t0 = a.split * a.tps;
    a.t1 = min(a.t0 + a.tps, a.ntiles);
    return a;
  };
  if (ct == 0) s_pre = 0;

  // act[m][0..K) = rmsnorm(src[m]) * nw, one rounding (src rows of stride K).
  auto norm_prologue = [&](const bf16* const* src_rows, const bf16* nw, int K) {
    float ss[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) ss[m] = 0.f;
    for (int k = ct * 8; k < K; k += kC * 32 * 8) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < p.B) {
          float f[8];
          unpack16<bf16>(__ldcg(reinterpret_cast<const uint4*>(src_rows[m] + k)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss[m] = fmaf(f[e], f[e], ss[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float v = warp_sum(ss[m]);
      if (lane == 0) red[warp * 4 + m] = v;
    }
    csync();
    float inv[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < kC; ++i) t += red[i * 4 + m];
      inv[m] = rsqrtf(t / (float)K + p.eps);
    }
    for (int k = ct * 8; k < K; k += kC * 32 * 8) {
      float wf[8];
      unpack16<bf16>(*reinterpret_cast<const uint4*>(nw + k), wf);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < p.B) {
          float f[8];
          unpack16<bf16>(__ldcg(reinterpret_cast<const uint4*>(src_rows[m] + k)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = f[e] * inv[m] * wf[e];
          *reinterpret_cast<uint4*>(act + (size_t)m * (K + kActPad) + k) = pack16<bf16>(f);
        }
      }
    }
    csync();
  };

  // One weight phase on the tensor cores (mma.sync m16n8k16, bf16 operands,
  // fp32 accumulation).  M is the token (A rows g < B; the rest are zero), N
  // the R rows of a stage, K this warp's eighth of the stage's columns.  Lane
  // (g = lane / 4, t = lane % 4) loads 16 bytes of weight row g and 16 bytes of
  // token g's activation at the same columns: since a dot product may sum its
  // terms in any order, those eight columns feed two MMAs directly (one column
  // permutation shared by both operands).  Each warp keeps its partial sums
  // of the group in its own slice of the group's accumulator (summing its kb
  // column blocks in order) and signals `posted` after the group's last
  // column block; the epilogue warp then adds the kC slices of row r, token m
  // in warp order -- a fixed summation order, so every step is
  // bit-reproducible.
  auto gemv_phase = [&](const WPhase& wp) {
    const int K = wp.K, KT = wp.KT, kb = wp.kb, R = wp.R;
    const int ns = (wp.ge - wp.gb) * kb;
    const int kw = KT / kC;  // columns per warp, a multiple of 32
    const int g8 = lane >> 2, t4 = lane & 3;
    const bool act_ok = g8 < p.B;
    const bf16* act_row = act + (size_t)g8 * (K + kActPad) + warp * kw + 8 * t4;
    int grp = wp.gb, kblk = -1;
    for (int t = 0; t < ns; ++t) {
      const int slot = r_slot;
      const uint32_t par = r_par;
      if (++r_slot == RING) {
        r_slot = 0;
        r_par ^= 1u;
      }
      if (++kblk == kb) {
        kblk = 0;
        ++grp;
      }
      const int ai = a_slot;
      if (kblk == kb - 1) a_slot = a_slot + 1 == NACC ? 0 : a_slot + 1;
      const int rows = min(R, wp.N - grp * R);
      if (!mwait(&full[slot], par) && lane == 0) atomicOr(p.err, 2);
      // four independent accumulator chains, summed in a fixed order
      float c[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) c[a][0] = c[a][1] = c[a][2] = c[a][3] = 0.f;
      {
        const uint8_t* wr = ring + (size_t)slot * kSlot + (size_t)g8 * wp.stride +
                            (size_t)(warp * kw + 8 * t4) * 2;
        const bf16* ar = act_row + (size_t)kblk * KT;
        const bool wok = g8 < rows;
        const uint4 z = make_uint4(0, 0, 0, 0);
        if (kw == 192) {  // K = 1536 in one block: all loads first, then the MMAs
          uint4 wv[6], av[6];
#pragma unroll
          for (int i = 0; i < 6; ++i) wv[i] = wok ? *reinterpret_cast<const uint4*>(wr + 64 * i) : z;
#pragma unroll
          for (int i = 0; i < 6; ++i) av[i] = act_ok ? *reinterpret_cast<const uint4*>(ar + 32 * i) : z;
#pragma unroll
          for (int i = 0; i < 6; ++i) {
            mma_bf16_16816(c[(i & 1) * 2], av[i].x, av[i].y, wv[i].x, wv[i].y);
            mma_bf16_16816(c[(i & 1) * 2 + 1], av[i].z, av[i].w, wv[i].z, wv[i].w);
          }
        } else {
          const int nk = kw / 32;
#pragma unroll 2
          for (int i = 0; i < nk; i += 2) {
            const bool two = i + 1 < nk;
            const uint4 wv0 = wok ? *reinterpret_cast<const uint4*>(wr + 64 * i) : z;
            const uint4 av0 = act_ok ? *reinterpret_cast<const uint4*>(ar + 32 * i) : z;
            const uint4 wv1 = wok && two ? *reinterpret_cast<const uint4*>(wr + 64 * i + 64) : z;
            const uint4 av1 = act_ok && two ? *reinterpret_cast<const uint4*>(ar + 32 * i + 32) : z;
            mma_bf16_16816(c[0], av0.x, av0.y, wv0.x, wv0.y);
            mma_bf16_16816(c[1], av0.z, av0.w, wv0.z, wv0.w);
            mma_bf16_16816(c[2], av1.x, av1.y, wv1.x, wv1.y);
            mma_bf16_16816(c[3], av1.z, av1.w, wv1.z, wv1.w);
          }
        }
      }
      // lane (g, t): token g's partial sums of rows 2t and 2t + 1
      float* acc = acc_s + ai * (kC * 32);
      if (act_ok && 2 * t4 < R) {
        float* mine = acc + warp * 32 + (2 * t4) * 4 + g8;
        const float s0 = (c[0][0] + c[1][0]) + (c[2][0] + c[3][0]);
        const float s1 = (c[0][1] + c[1][1]) + (c[2][1] + c[3][1]);
        mine[0] = kblk == 0 ? s0 : mine[0] + s0;
        mine[4] = kblk == 0 ? s1 : mine[4] + s1;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[slot]);
        // the release orders this warp's partial sums before the epilogue
        // warp's reads
        if (kblk == kb - 1) mbar_arrive(&posted[ai]);
      }
    }
    gs += ns;
  };

  // Epilogue operands of this CTA's rows, staged in shared memory (visible
  // after the next consumer barrier): q/k/v biases and the RoPE cos/sin of
  // each pair for each token; the residual rows for the o and down phases
  // (afterwards kept current by this CTA's own epilogues, as the o and down
  // phases split their rows alike).
  auto stage_qkv = [&](const WPhase& wp, int l, bool rope_too) {
    const int row_lo = wp.gb * wp.R, nrows = min(wp.ge * wp.R, wp.N) - row_lo;
    const bf16* bias = reinterpret_cast<const bf16*>(p.layers[l].bqkv);
    for (int idx = ct; idx < nrows * 4; idx += kC * 32) {
      const int i = idx >> 2, m = idx & 3, n = row_lo + i;
      if (m == 0) e_bias[i] = to_f(bias[n]);
      if (rope_too && (i & 1) == 0 && m < p.B && n / p.hd < p.nh + p.nkv)
        e_cs[(i >> 1) * 4 + m] = p.rope[(size_t)p.lens[m] * (p.hd >> 1) + ((n % p.hd) >> 1)];
    }
  };
  auto stage_x = [&](const WPhase& wp) {
    const int row_lo = wp.gb * wp.R, nrows = min(wp.ge * wp.R, wp.N) - row_lo;
    for (int idx = ct; idx < nrows * 4; idx += kC * 32) {
      const int i = idx >> 2, m = idx & 3;
      if (m < p.B) e_x[i * 4 + m] = __bfloat162float(__ldcg(X + (size_t)m * p.H + row_lo + i));
    }
  };

  for (int ph = 0; ph < nph; ++ph) {
    const int kind = phase_kind(p, ph);
    const int l = ph / 5;
    // ---- wait until every CTA finished the previous phase
    if (ph > 0) {
      if (ct == 0) {
        const uint64_t t0 = gtimer();
        while (ld_acquire(&p.sync[ph - 1]) < ARRIVALS) {
          if (gtimer() - t0 > kDeadlineNs) {
            atomicOr(p.err, 2);
            break;
          }
        }
        if (kind == PH_ATTN) fence_proxy_async_global();  // K/V rows written by QKV, read by TMA
      }
      csync();
    }
    if (p.trace && ct == 0) {
      const unsigned long long t = gtimer();
      atomicMax(&p.trace[ph * 4 + 3], t);
      if (bid == 0) p.trace[ph * 4 + 1] = t;
    }

    if (kind == PH_QKV) {
      // Prefetch the first tiles of this CTA's first attention item of the
      // layer: tiles below the new position were written by earlier steps.
      if (ct == 0) {
        s_pre = 0;
        if (bid < p.B * p.nkv * p.nsplit) {
          const AItem a = attn_geom(bid);
          const int old_end = (a.L - 1) / kAT;
          for (int q = 0; q < 2 && a.t0 + q < a.t1 && a.t0 + q < old_end; ++q) {
            tile_issue(l, a.b, a.gq, a.t0 + q, ac + q);
            s_pre = q + 1;
          }
        }
      }
      const bf16* rows_[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) rows_[m] = X + (size_t)m * p.H;
      if (l == 0 && p.embed_in) {
        // Layer 0 reads the embedding rows directly; CTA 0 also writes them
        // to the residual stream.  An id outside the vocabulary sets bit 0
        // of the error word and reads row 0 (the step's results are then
        // undefined and the caller is told by q2_model_check_error).
        const bf16* E = reinterpret_cast<const bf16*>(p.embed);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < p.B) {
            long long id = p.ids[m];
            if (id < 0 || id >= p.V) {
              if (ct == 0 && bid == 0) atomicOr(p.err, 1);
              id = 0;
            }
            rows_[m] = E + (size_t)id * p.H;
          }
        }
        if (bid == 0) {
          for (int k = ct * 8; k < p.H; k += kC * 32 * 8)
#pragma unroll
            for (int m = 0; m < MT; ++m)
              if (m < p.B)
                *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(p.x) + (size_t)m * p.H + k) =
                    *reinterpret_cast<const uint4*>(rows_[m] + k);
        }
      }
      WPhase wp;
      weight_phase(p, ph, bid, G, wp);
      stage_qkv(wp, l, l == 0);  // RoPE cos/sin depend on the positions only
      norm_prologue(rows_, reinterpret_cast<const bf16*>(p.layers[l].in_norm), p.H);
      gemv_phase(wp);
    } else if (kind == PH_ATTN) {
      const int items = p.B * p.nkv * p.nsplit;
      for (int item = bid; item < items; item += G) {
        const AItem a = attn_geom(item);
        const int split = a.split, b = a.b, gq = a.gq, L = a.L, ntiles = a.ntiles, tps = a.tps;
        const int t0 = a.t0, t1 = a.t1;
        if (t0 >= t1) continue;
        auto issue = [&](int t, int li) { tile_issue(l, b, gq, t, li); };
        if (ct == 0) {
          const int pre = item == bid ? s_pre : 0;
          for (int q = pre; q < 2 && t0 + q < t1; ++q) issue(t0 + q, ac + q);
        }
        const bf16* qrow = reinterpret_cast<const bf16*>(p.qb) + (size_t)b * p.qd + (size_t)gq * G_q * kHD;
        const float qscale = p.scale * kLog2e;
        for (int i = ct; i < G_q * kHD; i += kC * 32)
          qs[i] = __bfloat162float(__ldcg(qrow + i)) * qscale;
        if (ct < kAGMax) {
          ms[ct] = -INFINITY;
          ls[ct] = 0.f;
        }
        csync();
        const int dp = ct & 63, hg = ct >> 6;  // PV: dims (2dp, 2dp+1); heads hg, hg+4
        float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        for (int t = t0; t < t1; ++t) {
          const int li = ac + (t - t0);
          const int stg = li & 1;
          if (!mwait(&abar[stg], (uint32_t)((li >> 1) & 1)) && lane == 0) atomicOr(p.err, 2);
          const uint8_t* kt = tiles + (size_t)stg * 2 * kTileBytes;
          const uint8_t* vt = kt + kTileBytes;
          const int jn = min(kAT, L - t * kAT);
          {
            const int j = ct & 63;
            float sc[2] = {0.f, 0.f};
#pragma unroll
            for (int bx = 0; bx < kHD / 64; ++bx) {
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                float kf[8];
                unpack16<bf16>(*reinterpret_cast<const uint4*>(kt + bx * 8192 + swz(j, c * 8)), kf);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                  const int hh = hg + 4 * i;
                  if (hh < G_q) {
                    const float* qh = qs + hh * kHD + bx * 64 + c * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) sc[i] = fmaf(qh[e], kf[e], sc[i]);
                  }
                }
              }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int hh = hg + 4 * i;
              if (hh < G_q) S[hh * kAT + j] = (j < jn) ? sc[i] : -INFINITY;
            }
          }
          csync();
          if (warp < G_q) {
            const int hh = warp;
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
          csync();
          {
            const int bx = (2 * dp) >> 6, cc = (2 * dp) & 63;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int hh = hg + 4 * i;
              if (hh < G_q) {
                acc[i][0] *= al[hh];
                acc[i][1] *= al[hh];
              }
            }
            for (int j = 0; j < jn; ++j) {
              const uint32_t wv = *reinterpret_cast<const uint32_t*>(vt + bx * 8192 + swz(j, cc));
              const float v0 = __uint_as_float(wv << 16), v1 = __uint_as_float(wv & 0xffff0000u);
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const int hh = hg + 4 * i;
                if (hh < G_q) {
                  const float pj = S[hh * kAT + j];
                  acc[i][0] = fmaf(pj, v0, acc[i][0]);
                  acc[i][1] = fmaf(pj, v1, acc[i][1]);
                }
              }
            }
          }
          csync();
          if (ct == 0 && t + 2 < t1) issue(t + 2, li + 2);
        }
        ac += t1 - t0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int hh = hg + 4 * i;
          if (hh < G_q) {
            const size_t pidx = ((size_t)b * p.nh + gq * G_q + hh) * p.nsplit + split;
            p.part_o[pidx * kHD + 2 * dp] = acc[i][0];
            p.part_o[pidx * kHD + 2 * dp + 1] = acc[i][1];
          }
        }
        if (ct < G_q) {
          const size_t pidx = ((size_t)b * p.nh + gq * G_q + ct) * p.nsplit + split;
          p.part_ml[2 * pidx] = ms[ct];
          p.part_ml[2 * pidx + 1] = ls[ct];
        }
        // ---- the last of the nact non-empty splits of (b, gq) merges them:
        // o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, into att (bf16)
        const int nact = (ntiles + tps - 1) / tps;
        __threadfence();
        csync();
        if (ct == 0) {
          unsigned* ticket = p.sync + 5 * p.L + 2 + b * p.nkv + gq;
          s_last_merge = (atomicAdd(ticket, 1u) == (unsigned)nact - 1);
          if (s_last_merge) *ticket = 0u;  // ready for the next layer
        }
        csync();
        if (s_last_merge) {
          __threadfence();
          float* wts = S;  // [G_q][nact] (nact <= 64)
          for (int i = ct; i < G_q * nact; i += kC * 32) {
            const int hh = i / nact, sp = i % nact;
            const size_t pidx = ((size_t)b * p.nh + gq * G_q + hh) * p.nsplit + sp;
            qs[i] = __ldcg(p.part_ml + 2 * pidx);      // m (qs is free now)
            wts[i] = __ldcg(p.part_ml + 2 * pidx + 1);  // l
          }
          csync();
          if (ct < G_q) {
            float Mx = -INFINITY;
            for (int sp = 0; sp < nact; ++sp) Mx = fmaxf(Mx, qs[ct * nact + sp]);
            float den = 0.f;
            for (int sp = 0; sp < nact; ++sp) {
              const float e = exp2f(qs[ct * nact + sp] - Mx);
              qs[ct * nact + sp] = e;
              den = fmaf(wts[ct * nact + sp], e, den);
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
            for (int sp = 0; sp < nact; ++sp) wts[ct * nact + sp] = qs[ct * nact + sp] * inv;
          }
          csync();
          for (int e = ct; e < G_q * kHD; e += kC * 32) {
            const int hh = e / kHD, d = e % kHD;
            const float* po = p.part_o + (((size_t)b * p.nh + gq * G_q + hh) * p.nsplit) * kHD + d;
            const float* wv = wts + hh * nact;
            float o0 = 0.f, o1 = 0.f;
            int sp = 0;
            for (; sp + 1 < nact; sp += 2) {
              o0 = fmaf(wv[sp], __ldcg(po + (size_t)sp * kHD), o0);
              o1 = fmaf(wv[sp + 1], __ldcg(po + (size_t)(sp + 1) * kHD), o1);
            }
            if (sp < nact) o0 = fmaf(wv[sp], __ldcg(po + (size_t)sp * kHD), o0);
            reinterpret_cast<bf16*>(p.att)[(size_t)b * p.qd + (size_t)(gq * G_q + hh) * kHD + d] =
                from_f<bf16>(o0 + o1);
          }
        }
        csync();
      }
    } else if (kind == PH_O) {
      WPhase wp;
      weight_phase(p, ph, bid, G, wp);
      if (l == 0) stage_x(wp);
      const bf16* A = reinterpret_cast<const bf16*>(p.att);
      for (int k = ct * 8; k < p.qd; k += kC * 32 * 8)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < p.B)
            *reinterpret_cast<uint4*>(act + (size_t)m * (p.qd + kActPad) + k) =
                __ldcg(reinterpret_cast<const uint4*>(A + (size_t)m * p.qd + k));
      csync();
      gemv_phase(wp);
    } else if (kind == PH_GU) {
      const bf16* rows_[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) rows_[m] = X + (size_t)m * p.H;
      norm_prologue(rows_, reinterpret_cast<const bf16*>(p.layers[l].post_norm), p.H);
      WPhase wp;
      weight_phase(p, ph, bid, G, wp);
      gemv_phase(wp);
    } else if (kind == PH_DOWN) {
      const bf16* Sv = reinterpret_cast<const bf16*>(p.s);
      for (int k = ct * 8; k < p.I; k += kC * 32 * 8)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < p.B)
            *reinterpret_cast<uint4*>(act + (size_t)m * (p.I + kActPad) + k) =
                __ldcg(reinterpret_cast<const uint4*>(Sv + (size_t)m * p.I + k));
      csync();
      WPhase wp;
      weight_phase(p, ph, bid, G, wp);
      gemv_phase(wp);
    } else {  // PH_HEAD
      const bf16* rows_[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) rows_[m] = X + (size_t)m * p.H;
      norm_prologue(rows_, reinterpret_cast<const bf16*>(p.final_norm), p.H);
      WPhase wp;
      weight_phase(p, ph, bid, G, wp);
      gemv_phase(wp);
    }

    // ---- this CTA is done with the phase
    if (kind == PH_QKV) fence_proxy_async_global();  // new K/V rows are read by TMA next
    csync();
    if (ct == 0) {
      if (p.trace) {
        const unsigned long long t = gtimer();
        atomicMax(&p.trace[ph * 4 + 0], t);
        if (bid == 0) p.trace[ph * 4 + 2] = t;
      }
      // release: this CTA's writes of the phase (ordered before by the CTA
      // barrier) are visible to whoever acquires the counter
      s_flag = atom_add_release(&p.sync[ph], 1u) == ARRIVALS - 1 && ph == nph - 1;
    }
    csync();
  }

  // ---- drain: every copy this CTA issued has landed before it exits (the
  // waits only block if an earlier bounded wait gave up)
  if (ct == 0) {
    for (int sl = 0; sl < RING; ++sl)
      if (gs > sl) mwait(&full[sl], (uint32_t)(((gs - 1 - sl) / RING) & 1));
    for (int st = 0; st < 2; ++st)
      if (ac > st) mwait(&abar[st], (uint32_t)(((ac - 1 - st) / 2) & 1));
  }

  // ---- the last arrival of the last phase wraps up the step
  if (s_flag) wrap_up(ct);
}

// ======================================================================
bool pdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd) {
  if (hd != kHD || nkv <= 0 || nh % nkv != 0 || nh / nkv > kAGMax || nh > kNHMax) return false;
  if (qkvd % 2 || V <= 0) return false;
  // every K splits into column blocks of a multiple of 256 that fit a slot
  for (int K : {H, qd, I})
    if (phase_kblocks(K, 8) == 0 || phase_kblocks(K, 4) == 0) return false;
  const PGeo g = make_geo(kPMaxBatch, I > H ? I : H);
  return g.ring >= 2 && g.total <= kSmemMax;
}

size_t pdecode_sync_words(int L) { return (size_t)5 * L + 2 + kPMaxBatch * 16; }

template <int MT>
static q2_status pdecode_launch(const PDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                cudaStream_t st) {
  const int actw = p.I > p.H ? (p.I > p.qd ? p.I : p.qd) : (p.H > p.qd ? p.H : p.qd);
  const PGeo g = make_geo(MT, actw);
  if (g.ring < 2 || g.total > kSmemMax) {
    set_error("persistent decode: shared memory plan does not fit");
    return Q2_ERR_SHAPE;
  }
  const int G = num_sms();
  for (int N : {p.qkvd, p.H}) {  // rows per CTA with staged epilogue operands
    const int R = phase_rows(N, G);
    if ((N / R + G) / G * R > kEpiRows) {
      set_error("persistent decode: too many rows per CTA for this device");
      return Q2_ERR_SHAPE;
    }
  }
  Q2_CUDA_TRY(cudaFuncSetAttribute(pdecode_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)g.total));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = g.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, pdecode_kernel<MT>, p, g, kmap, vmap);
  if (e != cudaSuccess) {
    set_error(std::string("persistent decode launch: ") + cudaGetErrorString(e));
    return Q2_ERR_CUDA;
  }
  return Q2_OK;
}

q2_status launch_pdecode(const PDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t st) {
  if (p.B < 1 || p.B > kPMaxBatch || p.nsplit < 1 || p.nsplit > kSplitMax) {
    set_error("persistent decode: batch or split count out of range");
    return Q2_ERR_SHAPE;
  }
  if (p.B == 1) return pdecode_launch<1>(p, kmap, vmap, st);
  if (p.B == 2) return pdecode_launch<2>(p, kmap, vmap, st);
  return pdecode_launch<4>(p, kmap, vmap, st);
}

}  // namespace q2
