// sdecode.cu -- the batch-1 streaming decode step (see sdecode.h).
//
// Numerics are those of the operator-by-operator path: every operator's
// output is rounded to bf16 where the operator would write it back (the
// RMSNorm output, each linear output, the RoPE outputs, the SwiGLU output,
// each residual add); dot products and softmax run in fp32.
#include <limits.h>

#include "common.cuh"
#include "sdecode.h"
#include "tma.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kCW = 8;                 // consumer warps
constexpr int kCT = kCW * 32;          // consumer threads
constexpr int kThreads = kCT + 32;     // + the producer warp
constexpr int kSB = 24576;             // weight ring slot: 8 rows of K = 1536, or one down row
constexpr int kAT = 64;                // attention keys per tile
constexpr int kHD = 128;               // head dim of this kernel
constexpr int kTile = kAT * kHD * 2;   // one K (or V) tile
constexpr int kAGMax = 8;              // query heads per kv head
constexpr int kYMax = 256;             // rows per CTA of a short-row phase (parked row results)
constexpr int kDMax = 64;              // rows per CTA of the o and down phases
constexpr int kQMax = 64;              // q/k/v rows per CTA (staged epilogue operands)
constexpr int kSplitMax = 64;
constexpr int kLMax = 128;             // layers (the layer table sits in shared memory)
constexpr size_t kSmemMax = 232448;    // 227 KB per CTA
constexpr float kLog2e = 1.4426950408889634f;

enum { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_GU = 3, PH_DOWN = 4, PH_HEAD = 5 };

// s_flags slots
enum { F_LAST = 0, F_MERGE = 1, F_PRE = 2, F_STALE = 3, F_LEN = 4 };

__host__ __device__ inline size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared-memory map (offsets from a 1024-byte aligned base: the attention
// tiles are 128-byte-swizzled TMA boxes).
struct SLay {
  size_t tiles, ring, layers, wts, mraw, yrow, part, xres, ebias, ecs, mlw, amv, ami, bars, flags, total;
};

__host__ __device__ inline SLay slayout(int ring, int L) {
  SLay Y;
  size_t o = 0;
  Y.tiles = o;  // [2 stages][K | V] tiles; the per-warp attention partials between items
  o += 4 * (size_t)kTile;
  Y.ring = o;
  o += (size_t)ring * kSB;
  Y.layers = o;  // [L] layer weight pointers
  o = up(o + (size_t)L * sizeof(PLayer), 16);
  Y.wts = o;  // [kAGMax][kSplitMax] split weights of the merge
  o += (size_t)kAGMax * kSplitMax * 4;
  Y.mraw = o;  // [kAGMax][kSplitMax] split maxima of the merge
  o += (size_t)kAGMax * kSplitMax * 4;
  Y.yrow = o;  // [kYMax] row results of a short-row phase
  o += (size_t)kYMax * 4;
  Y.part = o;  // [kCW][kDMax] per-warp column-slice sums of the down rows
  o += (size_t)kCW * kDMax * 4;
  Y.xres = o;  // [kDMax] this CTA's rows of the residual stream
  o += (size_t)kDMax * 4;
  Y.ebias = o;  // [kQMax] q/k/v bias of this CTA's rows
  o += (size_t)kQMax * 4;
  Y.ecs = o;  // [kQMax / 2] RoPE (cos, sin) of this CTA's row pairs
  o += (size_t)kQMax / 2 * 8;
  Y.mlw = o;  // [kCW][kAGMax][2] per-warp attention max and sum
  o += (size_t)kCW * kAGMax * 2 * 4;
  Y.amv = o;  // [kCW] per-warp argmax values
  o += kCW * 4;
  Y.ami = up(o, 8);  // [kCW] per-warp argmax indices
  o = Y.ami + kCW * 8;
  Y.bars = up(o, 8);  // full[ring], empty[ring], abar[2]
  o = Y.bars + (2 * (size_t)ring + 2) * 8;
  Y.flags = o;
  o += 8 * 4;
  Y.total = o + 1024;  // slack for aligning the base
  return Y;
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

__device__ __forceinline__ unsigned atom_add_release(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Orders this thread's generic-proxy writes to shared memory before later
// async-proxy (TMA) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Consumer-warps-only barrier (the producer warp never joins it).
__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }

// mbarrier wait bounded by a deadline on the global timer; false if it ran out.
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, uint64_t deadline_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (;;) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (gtimer() - t0 > deadline_ns) return false;
  }
}

// Wait until a grid counter reaches `target`, bounded by the deadline; once
// some wait of this launch has run out (`gave_up` set) it gives up at once,
// so a stalled step ends after one deadline rather than one per phase.
__device__ __forceinline__ bool gwait(const unsigned* ctr, unsigned target, uint64_t deadline_ns,
                                      const unsigned* gave_up) {
  if (ld_acquire(ctr) >= target) return true;
  const uint64_t t0 = gtimer();
  for (unsigned it = 1;; ++it) {
    if (ld_acquire(ctr) >= target) return true;
    if ((it & 63u) == 0) {
      if (*reinterpret_cast<const volatile unsigned*>(gave_up)) return false;
      if (gtimer() - t0 > deadline_ns) return false;
    }
  }
}

__device__ __forceinline__ float silu_mul(float gv, float uv) { return uv * (gv / (1.0f + expf(-gv))); }

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

__device__ __forceinline__ int phase_kind(int L, int ph) { return ph == 5 * L ? PH_HEAD : ph % 5; }

// The weight rows a CTA streams in one phase: rows [r0, r1) of w [N][K], in
// stages of rs whole rows.  Rows are dealt out in contiguous blocks, in units
// of row pairs where the epilogue needs both members of a pair (RoPE
// partners, gate/up).  The o and down phases split their rows alike, so a CTA
// owns the same rows of the residual stream in both.
struct PW {
  const bf16* w;
  int K, r0, r1, rs;
};

__device__ __forceinline__ bool phase_w(const SDecode& p, const PLayer* layers, int ph, int bid, int G,
                                        PW& o) {
  const int kind = phase_kind(p.L, ph);
  if (kind == PH_ATTN) return false;
  const PLayer* lw = kind == PH_HEAD ? nullptr : &layers[ph / 5];
  int N, unit;
  switch (kind) {
    case PH_QKV: o.w = (const bf16*)lw->wqkv; N = p.qkvd; o.K = p.H; unit = 2; break;
    case PH_O: o.w = (const bf16*)lw->wo; N = p.H; o.K = p.qd; unit = 1; break;
    case PH_GU: o.w = (const bf16*)lw->wgu; N = 2 * p.I; o.K = p.H; unit = 2; break;
    case PH_DOWN: o.w = (const bf16*)lw->wd; N = p.H; o.K = p.I; unit = 1; break;
    default: o.w = (const bf16*)p.lm_head; N = p.V; o.K = p.H; unit = 1; break;
  }
  const long long units = N / unit;
  o.r0 = (int)(bid * units / G) * unit;
  o.r1 = (int)((bid + 1) * units / G) * unit;
  const int rb = o.K * 2;
  o.rs = rb <= kSB ? kSB / rb : 1;
  return true;
}

// Walks the stages a CTA streams, phase by phase (weight phases only).
struct Cursor {
  int ph, r;
  PW pw;
  __device__ void settle(const SDecode& p, const PLayer* layers, int bid, int G, int nph) {
    for (; ph < nph; ++ph) {
      if (!phase_w(p, layers, ph, bid, G, pw)) continue;
      r = pw.r0;
      if (pw.r0 < pw.r1) return;
    }
  }
  __device__ void start(const SDecode& p, const PLayer* layers, int bid, int G, int nph) {
    ph = 0;
    settle(p, layers, bid, G, nph);
  }
  __device__ bool valid(int nph) const { return ph < nph; }
  __device__ void next(const SDecode& p, const PLayer* layers, int bid, int G, int nph) {
    r += pw.rs;
    if (r < pw.r1) return;
    ++ph;
    settle(p, layers, bid, G, nph);
  }
  __device__ uint32_t bytes() const { return (uint32_t)(min(pw.rs, pw.r1 - r)) * pw.K * 2; }
  __device__ const bf16* src() const { return pw.w + (size_t)r * pw.K; }
};

}  // namespace

// ======================================================================
// NCH: 256-column chunks of a short row (K = H = qd = NCH * 256), held by each
// lane as NCH 16-byte pieces of the input vector; NQ: 16-byte pieces per lane
// of a warp's column slice of a long (down) row.
template <int NCH, int NQ>
__global__ void __launch_bounds__(kThreads, 1)
    sdecode_kernel(const SDecode p, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int RING = p.ring;
  const int L = p.L;
  const SLay Y = slayout(RING, L);
  uint8_t* tiles = smem + Y.tiles;
  uint8_t* ring = smem + Y.ring;
  PLayer* layers = reinterpret_cast<PLayer*>(smem + Y.layers);
  float* wts = reinterpret_cast<float*>(smem + Y.wts);
  float* mraw = reinterpret_cast<float*>(smem + Y.mraw);
  float* yrow = reinterpret_cast<float*>(smem + Y.yrow);
  float* part = reinterpret_cast<float*>(smem + Y.part);
  float* xres = reinterpret_cast<float*>(smem + Y.xres);
  float* ebias = reinterpret_cast<float*>(smem + Y.ebias);
  float2* ecs = reinterpret_cast<float2*>(smem + Y.ecs);
  float* mlw = reinterpret_cast<float*>(smem + Y.mlw);
  float* amv = reinterpret_cast<float*>(smem + Y.amv);
  long long* ami = reinterpret_cast<long long*>(smem + Y.ami);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Y.bars);
  uint64_t* empty = full + RING;
  uint64_t* abar = empty + RING;
  int* s_flags = reinterpret_cast<int*>(smem + Y.flags);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, bid = blockIdx.x;
  const int nph = p.run_head ? 5 * L + 1 : 5 * L;
  const uint64_t dl = p.deadline_ns;

  // the layer table in shared memory; the step's position
  for (int i = tid; i < L * (int)(sizeof(PLayer) / 8); i += kThreads)
    reinterpret_cast<unsigned long long*>(layers)[i] = reinterpret_cast<const unsigned long long*>(p.layers)[i];
  if (tid == 0) {
    for (int i = 0; i < RING; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kCW);
    }
    mbar_init(&abar[0], 1);
    mbar_init(&abar[1], 1);
    fence_mbar_init();
    s_flags[F_LEN] = __ldcg(p.lens);
    s_flags[F_PRE] = 0;
    s_flags[F_STALE] = -1;
  }
  __syncthreads();
  const int pos = s_flags[F_LEN];  // the new token's position
  const int alen = pos + 1;        // keys attended (the new token included)

  // ================================================================ producer
  // One lane walks this CTA's stages of the whole step and issues one bulk
  // copy per stage as soon as its slot is free; a second cursor runs
  // l2_ahead stages in front and pulls them into L2.
  if (warp == kCW) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      Cursor cur, ahead;
      cur.start(p, layers, bid, G, nph);
      ahead.start(p, layers, bid, G, nph);
      for (int i = 0; i < p.l2_ahead && ahead.valid(nph); ++i) {
        bulk_prefetch_l2(ahead.src(), ahead.bytes());
        ahead.next(p, layers, bid, G, nph);
      }
      int slot = 0;
      uint32_t par = 0;
      for (long long gs = 0; cur.valid(nph); ++gs) {
        if (gs >= RING && !bwait(&empty[slot], par ^ 1u, dl)) atomicOr(p.err, 2);
        const uint32_t bytes = cur.bytes();
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s_evict_first(ring + (size_t)slot * kSB, cur.src(), bytes, &full[slot], pol);
        if (p.l2_ahead > 0 && ahead.valid(nph)) {
          bulk_prefetch_l2(ahead.src(), ahead.bytes());
          ahead.next(p, layers, bid, G, nph);
        }
        cur.next(p, layers, bid, G, nph);
        if (++slot == RING) {
          slot = 0;
          par ^= 1u;
        }
      }
    }
    return;
  }

  // =============================================================== consumers
  const int ct = tid;
  const int Gq = p.nh / p.nkv;
  const int half = p.hd >> 1;
  const bf16* X = reinterpret_cast<const bf16*>(p.x);
  long long gs = 0;    // weight stages consumed
  int c_slot = 0;      // ring slot and parity of the next stage
  uint32_t c_par = 0;
  int ac = 0;          // attention tiles consumed
  float best_v = -INFINITY;  // lm_head: this warp's argmax over its rows
  long long best_i = LLONG_MAX;

  // The rows of the residual stream this CTA owns in the o and down phases,
  // kept here between its epilogues (x in global memory is the copy the
  // RMSNorm prologues read).
  {
    const int r0 = (int)((long long)bid * p.H / G), r1 = (int)((long long)(bid + 1) * p.H / G);
    const bf16* src = X;
    if (p.embed_in) {
      long long id = __ldcg(p.ids);
      if (id < 0 || id >= p.V) id = 0;
      src = reinterpret_cast<const bf16*>(p.embed) + (size_t)id * p.H;
    }
    for (int i = ct; i < r1 - r0; i += kCT) xres[i] = __bfloat162float(src[r0 + i]);
  }

  auto load_nw = [&](const void* nw, uint4 (&nwr)[NCH]) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) nwr[i] = __ldg(reinterpret_cast<const uint4*>(nw) + lane + 32 * i);
  };
  // xr = bf16(rmsnorm(src) * nw): every warp normalises the whole vector itself.
  auto norm_regs = [&](const bf16* src, const uint4 (&nwr)[NCH], float (&xr)[NCH][8]) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      unpack16<bf16>(__ldcg(reinterpret_cast<const uint4*>(src) + lane + 32 * i), xr[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(xr[i][e], xr[i][e], ss);
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)(NCH * 256) + p.eps);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      float wf[8];
      unpack16<bf16>(nwr[i], wf);
#pragma unroll
      for (int e = 0; e < 8; ++e) xr[i][e] = round_st<bf16>(xr[i][e] * inv * wf[e]);
    }
  };

  // The stages of one short-row phase: warp w takes rows w, w + 8, ... of each
  // stage; the row result goes to yrow (or, for the lm_head, to the logits).
  auto consume_short = [&](const PW& pw, bool head, const float (&xr)[NCH][8]) {
    for (int r = pw.r0; r < pw.r1; r += pw.rs, ++gs) {
      const int slot = c_slot;
      const uint32_t par = c_par;
      if (++c_slot == RING) {
        c_slot = 0;
        c_par ^= 1u;
      }
      const int n = min(pw.rs, pw.r1 - r);
      if (!bwait(&full[slot], par, dl) && lane == 0) atomicOr(p.err, 2);
      const uint8_t* st = ring + (size_t)slot * kSB;
      for (int rr = warp; rr < n; rr += kCW) {
        const uint4* wrow = reinterpret_cast<const uint4*>(st + (size_t)rr * pw.K * 2);
        float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          float wf[8];
          unpack16<bf16>(wrow[lane + 32 * i], wf);
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e & 3] = fmaf(wf[e], xr[i][e], a[e & 3]);
        }
        const float y = warp_sum((a[0] + a[1]) + (a[2] + a[3]));
        if (head) {
          const int row = r + rr;
          if (lane == 0) p.logits[row] = y;
          if (am_better(y, row, best_v, best_i)) {
            best_v = y;
            best_i = row;
          }
        } else if (lane == 0) {
          yrow[r + rr - pw.r0] = y;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  };

  // The stages of the down phase: one row per stage, warp w takes column
  // pieces [w * cpw, (w + 1) * cpw) of it.
  auto consume_long = [&](const PW& pw, const float (&xs)[NQ][8]) {
    const int cpw = pw.K / 8 / kCW;
    for (int r = pw.r0; r < pw.r1; r += pw.rs, ++gs) {
      const int slot = c_slot;
      const uint32_t par = c_par;
      if (++c_slot == RING) {
        c_slot = 0;
        c_par ^= 1u;
      }
      if (!bwait(&full[slot], par, dl) && lane == 0) atomicOr(p.err, 2);
      const uint4* wrow = reinterpret_cast<const uint4*>(ring + (size_t)slot * kSB) + warp * cpw;
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        if (lane + 32 * q < cpw) {
          float wf[8];
          unpack16<bf16>(wrow[lane + 32 * q], wf);
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e & 3] = fmaf(wf[e], xs[q][e], a[e & 3]);
        }
      }
      const float y = warp_sum((a[0] + a[1]) + (a[2] + a[3]));
      if (lane == 0) part[warp * kDMax + (r - pw.r0)] = y;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  };

  // ---- attention work items: (kv head, split) pairs; a split spans at least
  // two tiles (one per warp group) and its range follows from the length.
  struct AItem {
    int gq, split, ntiles, tps, t0, t1, nact;
  };
  auto attn_item = [&](int item) {
    AItem a;
    a.gq = item % p.nkv;
    a.split = item / p.nkv;
    a.ntiles = (alen + kAT - 1) / kAT;
    const int active = min(p.nsplit, (a.ntiles + 1) / 2);
    a.tps = (a.ntiles + active - 1) / active;
    a.t0 = a.split * a.tps;
    a.t1 = min(a.t0 + a.tps, a.ntiles);
    a.nact = (a.ntiles + a.tps - 1) / a.tps;
    return a;
  };
  // TMA load of K/V tile t of (layer l, kv head gq) into attention stage li & 1.
  auto tile_issue = [&](int l, int gq, int t, int li) {
    const int stg = li & 1;
    const int row_base = ((l * p.Bmax) * p.nkv + gq) * p.max_seq;
    uint8_t* kt = tiles + (size_t)stg * 2 * kTile;
    uint8_t* vt = kt + kTile;
    mbar_arrive_expect_tx(&abar[stg], 2 * kTile);
#pragma unroll
    for (int bx = 0; bx < kHD / 64; ++bx) {
      tma_load_2d(kt + bx * 8192, &kmap, bx * 64, row_base + t * kAT, &abar[stg]);
      tma_load_2d(vt + bx * 8192, &vmap, bx * 64, row_base + t * kAT, &abar[stg]);
    }
  };
  const int aitems = p.nkv * p.nsplit;

  for (int ph = 0; ph < nph; ++ph) {
    const int kind = phase_kind(L, ph);
    const int l = ph / 5;
    PW pw;
    phase_w(p, layers, ph, bid, G, pw);
    unsigned long long* ctr = p.ctrace ? p.ctrace + ((size_t)ph * G + bid) * 4 : nullptr;
    if (ctr && ct == 0) ctr[0] = gtimer();
    uint4 nwr[NCH];    // the RMSNorm weight pieces of this phase (loaded before its wait)
    float xr[NCH][8];  // short-row phases: this lane's pieces lane + 32 i of the input vector

    // ---- what does not depend on the previous phase, before waiting for it
    if (kind == PH_QKV) {
      load_nw(layers[l].in_norm, nwr);
      const bf16* bias = reinterpret_cast<const bf16*>(layers[l].bqkv);
      for (int i = ct; i < pw.r1 - pw.r0; i += kCT) {
        const int n = pw.r0 + i;
        ebias[i] = __bfloat162float(__ldg(bias + n));
        if ((i & 1) == 0 && n / p.hd < p.nh + p.nkv)
          ecs[i >> 1] = __ldg(p.rope + (size_t)pos * half + ((n % p.hd) >> 1));
      }
      // the first two tiles of this CTA's first attention item of the layer;
      // the tile holding the new position is patched once its row exists
      if (ct == 0) {
        s_flags[F_PRE] = 0;
        s_flags[F_STALE] = -1;
        if (bid < aitems) {
          const AItem a = attn_item(bid);
          for (int q = 0; q < 2 && a.t0 + q < a.t1; ++q) {
            tile_issue(l, a.gq, a.t0 + q, ac + q);
            if (a.t0 + q == a.ntiles - 1) s_flags[F_STALE] = ac + q;
            s_flags[F_PRE] = q + 1;
          }
        }
      }
    } else if (kind == PH_GU) {
      load_nw(layers[l].post_norm, nwr);
    } else if (kind == PH_HEAD) {
      load_nw(p.final_norm, nwr);
    }

    // ---- wait until every CTA has finished the previous phase
    if (ph > 0) {
      if (ct == 0) {
        const unsigned target = (unsigned)G + (ph - 1 == p.stall_phase ? 1u : 0u);
        unsigned* gave_up = p.sync + 5 * L + 1 + L * p.nkv;
        if (!gwait(&p.sync[ph - 1], target, dl, gave_up)) {
          atomicOr(p.err, 2);
          atomicExch(gave_up, 1u);
        }
        __threadfence();
        if (kind == PH_ATTN) fence_proxy_async_global();  // new K/V rows, read next by TMA
      }
      csync();
    }
    if (p.trace && ct == 0) {
      const unsigned long long t = gtimer();
      atomicMax(&p.trace[ph * 4 + 3], t);
      if (bid == 0) p.trace[ph * 4 + 1] = t;
    }
    if (ctr && ct == 0) ctr[1] = gtimer();

    if (kind == PH_ATTN) {
      // Tensor-core attention over each tile: warp (grp, wq) takes keys
      // [16 wq, 16 wq + 16) and output dims [64 grp, 64 grp + 64): scores
      // q_h . k_j by mma.sync (the kv head's query heads on M, keys on N, head
      // dims on K; both groups compute them), online softmax in fp32, P . V by
      // mma.sync (P in a bf16 high and low part) for the group's dims.  The
      // four warps of a group are merged in shared memory, then the splits by
      // the last split to finish.
      const int grp = warp >> 2, wq = warp & 3;
      const int fr = lane >> 2, fc = lane & 3;  // mma fragment coordinates
      const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: lane addresses row mr of matrix mi
      const float sl2 = p.scale * kLog2e;
      for (int item = bid; item < aitems; item += G) {
        const AItem a = attn_item(item);
        if (a.t0 >= a.t1) continue;
        const int nt = a.t1 - a.t0;
        const int pre = item == bid ? s_flags[F_PRE] : 0;
        const int stale = item == bid ? s_flags[F_STALE] : -1;
        if (ct == 0)
          for (int q = pre; q < 2 && q < nt; ++q) tile_issue(l, a.gq, a.t0 + q, ac + q);
        // the new K/V row (for a tile loaded before it was written): fetched
        // now, stored into the tile once the tile has landed
        uint4 nrow = make_uint4(0u, 0u, 0u, 0u);
        if (stale >= 0 && warp == 0) {
          const size_t off = (size_t)l * p.kv_layer_stride + ((size_t)a.gq * p.max_seq + pos) * kHD;
          const bf16* src = reinterpret_cast<const bf16*>(lane < 16 ? p.kc : p.vc) + off;
          nrow = __ldcg(reinterpret_cast<const uint4*>(src) + (lane & 15));
        }
        // A fragments of the query heads (bf16, unscaled); rows fr >= Gq are zero
        uint32_t qa[8][2];
        {
          const unsigned* qrow = reinterpret_cast<const unsigned*>(
              reinterpret_cast<const bf16*>(p.qb) + (size_t)(a.gq * Gq + (fr < Gq ? fr : 0)) * kHD);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            qa[kk][0] = fr < Gq ? __ldcg(qrow + 8 * kk + fc) : 0u;
            qa[kk][1] = fr < Gq ? __ldcg(qrow + 8 * kk + fc + 4) : 0u;
          }
        }
        float o[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        float m_run = -INFINITY, l_run = 0.f;
        for (int i = 0; i < nt; ++i) {
          const int li = ac + i, stg = li & 1;
          const int t = a.t0 + i;
          if (!bwait(&abar[stg], (uint32_t)((li >> 1) & 1), dl) && lane == 0) atomicOr(p.err, 2);
          uint8_t* tk = tiles + (size_t)stg * 2 * kTile;
          if (li == stale) {
            if (warp == 0) {
              const int r = pos - t * kAT, c = lane & 15;
              uint8_t* dst = tk + (lane < 16 ? 0 : kTile) + (c >> 3) * 8192 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
              *reinterpret_cast<uint4*>(dst) = nrow;
              fence_proxy_async_smem();
            }
            csync();
          }
          const uint32_t kt = smem_u32(tk);
          const uint32_t vt = kt + (uint32_t)kTile;
          // ---- scores of this warp's 16 keys: s0 keys +0..7, s1 keys +8..15
          float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
          {
            const int key = wq * 16 + ((mi >> 1) << 3) + mr;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const int dim = 16 * kk + ((mi & 1) << 3);
              uint32_t r0, r1, r2, r3;
              ldsm_x4(kt + (uint32_t)((dim >> 6) * 8192) + swz_off(key, dim & 63), r0, r1, r2, r3);
              mma16816(s0, qa[kk][0], qa[kk][1], r0, r1);
              mma16816(s1, qa[kk][0], qa[kk][1], r2, r3);
            }
          }
          // ---- online softmax for head fr over keys kb + 2fc, +1 and kb + 8 + 2fc, +1
          const int kb = t * kAT + wq * 16 + 2 * fc;
          float sc[4] = {s0[0] * sl2, s0[1] * sl2, s1[0] * sl2, s1[1] * sl2};
          if (kb >= alen) sc[0] = -INFINITY;
          if (kb + 1 >= alen) sc[1] = -INFINITY;
          if (kb + 8 >= alen) sc[2] = -INFINITY;
          if (kb + 9 >= alen) sc[3] = -INFINITY;
          float mloc = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
          mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
          mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
          const float mnew = fmaxf(m_run, mloc);
          const float msafe = mnew == -INFINITY ? 0.f : mnew;
          const float alpha = exp2f(m_run - msafe);
          float pr[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) pr[e] = exp2f(sc[e] - msafe);
          float psum = (pr[0] + pr[1]) + (pr[2] + pr[3]);
          psum += __shfl_xor_sync(0xffffffffu, psum, 1);
          psum += __shfl_xor_sync(0xffffffffu, psum, 2);
          l_run = l_run * alpha + psum;
          m_run = mnew;
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            o[n][0] *= alpha;
            o[n][1] *= alpha;
          }
          // P in two bf16 parts, hi = bf16(p) and lo = bf16(p - hi), so that the
          // probabilities keep ~16 significant bits through the bf16 MMA.
          float ph_[4], pl_[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            ph_[e] = __bfloat162float(__float2bfloat16_rn(pr[e]));
            pl_[e] = pr[e] - ph_[e];
          }
          const uint32_t pa0 = pack_bf16x2(ph_[0], ph_[1]), pa2 = pack_bf16x2(ph_[2], ph_[3]);
          const uint32_t pb0 = pack_bf16x2(pl_[0], pl_[1]), pb2 = pack_bf16x2(pl_[2], pl_[3]);
          // positions past the sequence hold stale cache rows (possibly not
          // finite): their V entries are zeroed, as 0 * inf would poison the sum
          const uint32_t vm0 = (kb < alen ? 0x0000ffffu : 0u) | (kb + 1 < alen ? 0xffff0000u : 0u);
          const uint32_t vm1 = (kb + 8 < alen ? 0x0000ffffu : 0u) | (kb + 9 < alen ? 0xffff0000u : 0u);
          // ---- O += P . V over the same 16 keys, the group's 64 dims, 16 (two
          // n8 tiles) per ldmatrix
          {
            const int key = wq * 16 + ((mi & 1) << 3) + mr;
#pragma unroll
            for (int nd = 0; nd < 4; ++nd) {
              const int dim = 64 * grp + 16 * nd + ((mi >> 1) << 3);
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
          csync();  // every warp is done with this stage
          if (ct == 0 && i + 2 < nt) tile_issue(l, a.gq, t + 2, li + 2);
        }
        ac += nt;

        // ---- the four warps of each group (max, sum, unnormalised output), merged;
        // the tile buffers are free now (every tile of the item was waited on)
        float* Ow = reinterpret_cast<float*>(tiles);  // [kCW][kAGMax][64]
        if (fr < Gq) {
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            float* dst = Ow + ((size_t)warp * kAGMax + fr) * 64 + 8 * n + 2 * fc;
            dst[0] = o[n][0];
            dst[1] = o[n][1];
          }
          if (fc == 0) {
            mlw[(warp * kAGMax + fr) * 2] = m_run;
            mlw[(warp * kAGMax + fr) * 2 + 1] = l_run;
          }
        }
        csync();
        const bool direct = a.nact == 1;
        for (int i = ct; i < Gq * kHD; i += kCT) {
          const int hh = i / kHD, d = i % kHD, w0 = 4 * (d >> 6);
          float M = -INFINITY;
#pragma unroll
          for (int w = w0; w < w0 + 4; ++w) M = fmaxf(M, mlw[(w * kAGMax + hh) * 2]);
          const float Ms = M == -INFINITY ? 0.f : M;
          float O = 0.f, Ls = 0.f;
#pragma unroll
          for (int w = w0; w < w0 + 4; ++w) {
            const float e = exp2f(mlw[(w * kAGMax + hh) * 2] - Ms);
            O = fmaf(e, Ow[((size_t)w * kAGMax + hh) * 64 + (d & 63)], O);
            Ls = fmaf(e, mlw[(w * kAGMax + hh) * 2 + 1], Ls);
          }
          if (direct) {
            reinterpret_cast<bf16*>(p.att)[(size_t)(a.gq * Gq + hh) * kHD + d] =
                __float2bfloat16_rn(Ls > 0.f ? O / Ls : 0.f);
          } else {
            const size_t pidx = (size_t)(a.gq * Gq + hh) * p.nsplit + a.split;
            p.part_o[pidx * kHD + d] = O;
            if (d == 0) {
              p.part_ml[2 * pidx] = M;
              p.part_ml[2 * pidx + 1] = Ls;
            }
          }
        }
        fence_proxy_async_smem();  // the tile buffer is a TMA destination again later
        if (!direct) {
          // ---- the last of the nact splits of this kv head merges them:
          // o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, in split order
          __threadfence();
          csync();
          if (ct == 0) {
            unsigned* ticket = p.sync + 5 * L + 1 + l * p.nkv + a.gq;
            s_flags[F_MERGE] = atomicAdd(ticket, 1u) == (unsigned)a.nact - 1;
          }
          csync();
          if (s_flags[F_MERGE]) {
            __threadfence();
            for (int i = ct; i < Gq * a.nact; i += kCT) {
              const int hh = i / a.nact, sp = i % a.nact;
              const size_t pidx = (size_t)(a.gq * Gq + hh) * p.nsplit + sp;
              mraw[hh * kSplitMax + sp] = __ldcg(p.part_ml + 2 * pidx);
              wts[hh * kSplitMax + sp] = __ldcg(p.part_ml + 2 * pidx + 1);
            }
            csync();
            if (ct < Gq) {
              float Mx = -INFINITY;
              for (int sp = 0; sp < a.nact; ++sp) Mx = fmaxf(Mx, mraw[ct * kSplitMax + sp]);
              const float Ms = Mx == -INFINITY ? 0.f : Mx;
              float den = 0.f;
              for (int sp = 0; sp < a.nact; ++sp) {
                const float e = exp2f(mraw[ct * kSplitMax + sp] - Ms);
                mraw[ct * kSplitMax + sp] = e;
                den = fmaf(wts[ct * kSplitMax + sp], e, den);
              }
              const float inv = den > 0.f ? 1.f / den : 0.f;
              for (int sp = 0; sp < a.nact; ++sp) wts[ct * kSplitMax + sp] = mraw[ct * kSplitMax + sp] * inv;
            }
            csync();
            for (int e = ct; e < Gq * kHD; e += kCT) {
              const int hh = e / kHD, d = e % kHD;
              const float* po = p.part_o + ((size_t)(a.gq * Gq + hh) * p.nsplit) * kHD + d;
              const float* wv = wts + hh * kSplitMax;
              float o0 = 0.f, o1 = 0.f;
              int sp = 0;
              for (; sp + 1 < a.nact; sp += 2) {
                o0 = fmaf(wv[sp], __ldcg(po + (size_t)sp * kHD), o0);
                o1 = fmaf(wv[sp + 1], __ldcg(po + (size_t)(sp + 1) * kHD), o1);
              }
              if (sp < a.nact) o0 = fmaf(wv[sp], __ldcg(po + (size_t)sp * kHD), o0);
              reinterpret_cast<bf16*>(p.att)[(size_t)(a.gq * Gq + hh) * kHD + d] = __float2bfloat16_rn(o0 + o1);
            }
          }
        }
        csync();
      }
    } else if (kind == PH_DOWN) {
      float xs[NQ][8];  // this lane's pieces of the warp's column slice of s
      const int cpw = pw.K / 8 / kCW;
      const uint4* sv = reinterpret_cast<const uint4*>(p.s) + warp * cpw;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        if (lane + 32 * q < cpw) {
          unpack16<bf16>(__ldcg(sv + lane + 32 * q), xs[q]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xs[q][e] = 0.f;
        }
      }
      consume_long(pw, xs);
    } else {  // the short-row phases: q/k/v, o, gate/up, lm_head
      if (kind == PH_O) {
#pragma unroll
        for (int i = 0; i < NCH; ++i)
          unpack16<bf16>(__ldcg(reinterpret_cast<const uint4*>(p.att) + lane + 32 * i), xr[i]);
      } else {
        const bf16* src = X;
        if (kind == PH_QKV && l == 0 && p.embed_in) {
          // layer 0 normalises the embedding row directly.  An id outside the
          // vocabulary sets bit 0 of the error word and reads row 0.
          long long id = __ldcg(p.ids);
          if (id < 0 || id >= p.V) {
            if (ct == 0 && bid == 0) atomicOr(p.err, 1);
            id = 0;
          }
          src = reinterpret_cast<const bf16*>(p.embed) + (size_t)id * p.H;
        }
        norm_regs(src, nwr, xr);
      }
      consume_short(pw, kind == PH_HEAD, xr);
    }

    // ---- phase epilogue from the parked row results and staged operands
    csync();
    if (ctr && ct == 0) ctr[2] = gtimer();
    if (kind == PH_QKV) {
      const size_t loff = (size_t)l * p.kv_layer_stride;
      for (int i = ct; 2 * i < pw.r1 - pw.r0; i += kCT) {
        const int n = pw.r0 + 2 * i;
        const int hs = n / p.hd, j = (n % p.hd) >> 1;
        const float va = round_st<bf16>(yrow[2 * i] + ebias[2 * i]);
        const float vb = round_st<bf16>(yrow[2 * i + 1] + ebias[2 * i + 1]);
        if (hs < p.nh + p.nkv) {
          const float2 cs = ecs[i];
          const bf16 ra = __float2bfloat16_rn(va * cs.x - vb * cs.y);
          const bf16 rb = __float2bfloat16_rn(vb * cs.x + va * cs.y);
          bf16* dst = hs < p.nh ? reinterpret_cast<bf16*>(p.qb) + (size_t)hs * p.hd
                                : reinterpret_cast<bf16*>(p.kc) + loff + ((size_t)(hs - p.nh) * p.max_seq + pos) * p.hd;
          dst[j] = ra;
          dst[j + half] = rb;
        } else {
          bf16* dst = reinterpret_cast<bf16*>(p.vc) + loff +
                      ((size_t)(hs - p.nh - p.nkv) * p.max_seq + pos) * p.hd;
          dst[j] = __float2bfloat16_rn(va);
          dst[j + half] = __float2bfloat16_rn(vb);
        }
      }
      fence_proxy_async_global();  // attention may read the new K/V rows by TMA
    } else if (kind == PH_O || kind == PH_DOWN) {
      bf16* xw = reinterpret_cast<bf16*>(p.x);
      for (int i = ct; i < pw.r1 - pw.r0; i += kCT) {
        float y;
        if (kind == PH_O) {
          y = yrow[i];
        } else {
          y = 0.f;
#pragma unroll
          for (int w = 0; w < kCW; ++w) y += part[w * kDMax + i];
        }
        const bf16 xn = __float2bfloat16_rn(xres[i] + round_st<bf16>(y));
        xw[pw.r0 + i] = xn;
        xres[i] = __bfloat162float(xn);
      }
    } else if (kind == PH_GU) {
      bf16* sw = reinterpret_cast<bf16*>(p.s);
      for (int i = ct; 2 * i < pw.r1 - pw.r0; i += kCT) {
        const float gv = round_st<bf16>(yrow[2 * i]), uv = round_st<bf16>(yrow[2 * i + 1]);
        sw[(pw.r0 >> 1) + i] = __float2bfloat16_rn(silu_mul(gv, uv));
      }
    } else if (kind == PH_HEAD) {
      if (lane == 0) {
        amv[warp] = best_v;
        ami[warp] = best_i;
      }
      csync();
      if (ct == 0) {
        float bv = -INFINITY;
        long long bi = LLONG_MAX;
        for (int w = 0; w < kCW; ++w)
          if (am_better(amv[w], ami[w], bv, bi)) {
            bv = amv[w];
            bi = ami[w];
          }
        p.am_val[bid] = bv;
        p.am_idx[bid] = bi;
      }
    }

    // ---- this CTA is done with the phase
    csync();
    if (ct == 0) {
      __threadfence();
      s_flags[F_LAST] = atom_add_release(&p.sync[ph], 1u) == (unsigned)G - 1 && ph == nph - 1;
      if (ctr) ctr[3] = gtimer();
      if (p.trace) {
        const unsigned long long t = gtimer();
        atomicMax(&p.trace[ph * 4 + 0], t);
        if (bid == 0) p.trace[ph * 4 + 2] = t;
      }
    }
  }

  // ---- drain: every copy this CTA issued has landed before it exits (the
  // waits only block if an earlier bounded wait gave up)
  if (ct == 0) {
    for (int sl = 0; sl < RING; ++sl)
      if (gs > sl) bwait(&full[sl], (uint32_t)(((gs - 1 - sl) / RING) & 1), dl);
    for (int st = 0; st < 2; ++st)
      if (ac > st) bwait(&abar[st], (uint32_t)(((ac - 1 - st) / 2) & 1), dl);
  }
  csync();

  // ---- the last arrival of the last phase wraps up the step: the token
  // (argmax over the CTAs' partials) and the length
  if (s_flags[F_LAST] && ct == 0) {
    __threadfence();
    if (p.run_head) {
      float bv = -INFINITY;
      long long bi = LLONG_MAX;
      for (int b = 0; b < G; ++b) {
        const float v = __ldcg(p.am_val + b);
        const long long i = __ldcg(reinterpret_cast<const long long*>(p.am_idx) + b);
        if (am_better(v, i, bv, bi)) {
          bv = v;
          bi = i;
        }
      }
      p.next[0] = bi;
    }
    p.lens[0] += 1;
  }
}

// ======================================================================
namespace {
constexpr int kNCH = 6;  // H = 1536
constexpr int kNQ = 5;   // ceil(I / 8 / kCW / 32) for I = 8960
}  // namespace

bool sdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd) {
  if (hd != kHD || nkv <= 0 || nh % nkv != 0 || nh / nkv > kAGMax || V <= 0) return false;
  if (H != kNCH * 256 || qd != H || qkvd % 2 != 0) return false;
  if (I % (8 * kCW) != 0 || (I / 8 / kCW + 31) / 32 != kNQ || I * 2 > kSB || I * 2 <= kSB / 2)
    return false;
  return true;
}

// phase counters [5L + 1], merge tickets [L][nkv], the launch's give-up word
size_t sdecode_sync_words(int L, int nkv) { return (size_t)5 * L + 1 + (size_t)L * nkv + 1; }

int sdecode_default_ring() { return 6; }

q2_status launch_sdecode(const SDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t st) {
  if (!sdecode_supported(p.H, p.I, p.V, p.nh, p.nkv, p.hd, p.qkvd, p.qd) || p.nsplit < 1 ||
      p.nsplit > kSplitMax || p.ring < 2 || p.L < 1 || p.L > kLMax) {
    set_error("streaming decode: unsupported shape");
    return Q2_ERR_SHAPE;
  }
  const SLay Y = slayout(p.ring, p.L);
  if (Y.total > kSmemMax) {
    set_error("streaming decode: the shared-memory plan does not fit");
    return Q2_ERR_SHAPE;
  }
  const int G = num_sms();
  // rows per CTA of the phases whose row results and operands sit in shared memory
  const long long qkv_rows = (long long)(p.qkvd / 2 + G - 1) / G * 2;
  const long long gu_rows = (long long)(p.I + G - 1) / G * 2;
  const long long o_rows = (p.H + G - 1) / G;
  if (qkv_rows > kQMax || gu_rows > kYMax || o_rows > kYMax || o_rows > kDMax) {
    set_error("streaming decode: too many rows per CTA for this device");
    return Q2_ERR_SHAPE;
  }
  auto kern = sdecode_kernel<kNCH, kNQ>;
  Q2_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Y.total));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Y.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, kmap, vmap);
  if (e != cudaSuccess) {
    set_error(std::string("streaming decode launch: ") + cudaGetErrorString(e));
    return Q2_ERR_CUDA;
  }
  return Q2_OK;
}

}  // namespace q2
