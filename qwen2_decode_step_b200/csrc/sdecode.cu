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

constexpr int kCW = 8;                 // consumer warps (two warpgroups)
constexpr int kCT = kCW * 32;          // consumer threads
constexpr int kThreads = kCT + 128;    // + the producer warpgroup (one warp of it streams)
// Registers: the block is launched with kLaunchRegs per thread (what 384
// threads and one block per SM allow: the register file of an SM sub-partition
// holds three warps at 168); the producer warpgroup hands most of its share to
// the consumer warpgroups.  The shares add up to the launch's total exactly.
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 56;
constexpr int kConsumerRegs = 224;
static_assert(kProducerRegs * 128 + kConsumerRegs * kCT == kLaunchRegs * kThreads,
              "the warpgroups' register shares must add up to the launch's");
constexpr int kSB = 24576;             // weight ring slot: 8 rows of K = 1536, or one down row
constexpr int kAT = 64;                // attention keys per tile
constexpr int kHD = 128;               // head dim of this kernel
constexpr int kTile = kAT * kHD * 2;   // one K (or V) tile
constexpr int kAGMax = 8;              // query heads per kv head
constexpr int kPS = 72;                // keys per row of the attention P buffers (64 + padding)
constexpr int kYMax = 256;             // rows per CTA of a short-row phase (parked row results)
constexpr int kDMax = 64;              // rows per CTA of the o and down phases
constexpr int kQMax = 64;              // q/k/v rows per CTA (staged epilogue operands)
constexpr int kHMax = 2048;            // hidden size (the staged input vector)
constexpr int kSplitMax = kSDecodeSplitMax;
constexpr size_t kSmemMax = 232448;    // 227 KB per CTA
constexpr float kLog2e = 1.4426950408889634f;

enum { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_GU = 3, PH_DOWN = 4, PH_HEAD = 5 };

__host__ __device__ inline size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared-memory map (offsets from a 1024-byte aligned base: the attention
// tiles are 128-byte-swizzled TMA boxes).  Every area but the weight ring and
// the layer table has a fixed size and sits at a compile-time offset; the ring
// (its depth is a launch parameter) and the layer table follow them.
namespace sl {
constexpr size_t kTiles = 0;  // [2 stages][K | V] tiles; the attention mergers' staged partials
constexpr size_t kYrow = kTiles + 4 * (size_t)kTile;           // [kYMax] row results of a short-row phase
constexpr size_t kPart = kYrow + (size_t)kYMax * 4;            // [kCW][kDMax] down-row column-slice sums
constexpr size_t kXres = kPart + (size_t)kCW * kDMax * 4;       // [kDMax] this CTA's residual rows
constexpr size_t kEbias = kXres + (size_t)kDMax * 4;           // [kQMax] q/k/v bias of this CTA's rows
constexpr size_t kEcs = kEbias + (size_t)kQMax * 4;            // [kQMax / 2] RoPE (cos, sin) per row pair
constexpr size_t kMlw = kEcs + (size_t)kQMax / 2 * 8;          // [128] attention: per-head rescale, merge weights
constexpr size_t kAmv = kMlw + (size_t)kCW * kAGMax * 2 * 4;   // [kCW] per-warp argmax values
constexpr size_t kAmi = kAmv + (size_t)kCW * 8;                // [kCW] per-warp argmax indices (8-aligned)
constexpr size_t kXbuf = kAmi + (size_t)kCW * 8;               // [kHMax] bf16: the phase's input vector
constexpr size_t kQst = kXbuf + (size_t)kHMax * 2;             // [kAGMax][kHD] bf16: one kv head's query heads
constexpr size_t kKvn = kQst + (size_t)kAGMax * kHD * 2;       // [2][kHD] bf16: its new K and V rows
constexpr size_t kAbar = kKvn + 2 * (size_t)kHD * 2;           // abar[2]
constexpr size_t kFlags = kAbar + 2 * 8;                       // [8] ints
constexpr size_t kRing = (kFlags + 8 * 4 + 1023) / 1024 * 1024;  // [ring][kSB] weight ring
static_assert(kAmi % 8 == 0 && kXbuf % 16 == 0 && kAbar % 8 == 0, "shared-memory alignment");
// the attention phase borrows: xbuf for the partial scores, yrow + part for P
// (high and low), mlw for the rescale and merge weights, the tiles for the
// merger's staged partials
static_assert(2 * kAT * kAGMax * 4 <= kHMax * 2, "attention scores");
static_assert(kPart == kYrow + (size_t)kYMax * 4 && 2 * kAGMax * kPS * 2 <= kYMax * 4 + kCW * kDMax * 4, "P");
static_assert(kAGMax + kSplitMax + 1 <= kCW * kAGMax * 2, "merge weights");
static_assert((size_t)kSplitMax * (kHD + 2) * 4 <= 4 * (size_t)kTile, "merger staging");
static_assert(kAT == 64 && kHD == 16 * kCW && kAGMax <= kCW, "attention work split");
}  // namespace sl

struct SLay {
  size_t ring, bars, layers, total;
};

__host__ __device__ inline SLay slayout(int ring, int L) {
  SLay Y;
  Y.ring = sl::kRing;
  Y.bars = Y.ring + (size_t)ring * kSB;  // full[ring], empty[ring]
  Y.layers = up(Y.bars + 2 * (size_t)ring * 8, 16);  // [L] layer weight pointers
  Y.total = Y.layers + (size_t)L * sizeof(PLayer) + 1024;  // + slack for aligning the base
  return Y;
}

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Orders this thread's generic-proxy writes to shared memory before later
// async-proxy (TMA) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Consumer-warps-only barrier (the producer warp never joins it).
__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }

// mbarrier wait bounded by a deadline on the global timer; false if it ran
// out.  With `gave_up` given, it also stops as soon as some wait of the launch
// has given up (the step's results are undefined by then).
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, uint64_t deadline_ns,
                                      const unsigned* gave_up = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (;;) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (gtimer() - t0 > deadline_ns) return false;
    if (gave_up && *reinterpret_cast<const volatile unsigned*>(gave_up) != 0u) return false;
  }
}

// ---------------------------------------------------------- tagged words
// A word is {u32 data, u32 tag}; 8-byte accesses are single-copy atomic, so a
// reader sees data and tag of the same store.  Stores and loads are volatile
// (no L1 caching): they meet in L2.
__device__ __forceinline__ void ll_put(uint64_t* w, uint32_t data, uint32_t tag) {
  const uint64_t v = ((uint64_t)tag << 32) | data;
  asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(w), "l"(v) : "memory");
}
// Two consecutive words (16-byte aligned) in one vector store.
__device__ __forceinline__ void ll_put2(uint64_t* w, uint32_t d0, uint32_t d1, uint32_t tag) {
  asm volatile("st.volatile.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(w), "r"(d0), "r"(tag), "r"(d1),
               "r"(tag)
               : "memory");
}

// Bounded polling of tagged words.  Once any wait of the launch has run out
// (`gave_up`), a poll that does not succeed at once gives up too, so a
// stalled step ends after one deadline rather than one per wait.
struct Poll {
  uint64_t deadline_ns;
  unsigned* gave_up;
  int* err;
  __device__ void fail() const {
    atomicOr(err, 2);
    atomicExch(gave_up, 1u);
  }
  __device__ bool stop(uint64_t t0) const {
    return *reinterpret_cast<volatile unsigned*>(gave_up) != 0u || gtimer() - t0 > deadline_ns;
  }
  // two consecutive words (16-byte aligned)
  __device__ uint2 get2(const uint64_t* w, uint32_t tag) const {
    uint32_t d0, t0_, d1, t1_;
    asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d0), "=r"(t0_), "=r"(d1), "=r"(t1_)
                 : "l"(w)
                 : "memory");
    if (t0_ == tag && t1_ == tag) return make_uint2(d0, d1);
    const uint64_t t0 = gtimer();
    for (unsigned it = 1;; ++it) {
      asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(d0), "=r"(t0_), "=r"(d1), "=r"(t1_)
                   : "l"(w)
                   : "memory");
      if (t0_ == tag && t1_ == tag) return make_uint2(d0, d1);
      if ((it & 15u) == 0 && stop(t0)) {
        fail();
        return make_uint2(d0, d1);
      }
    }
  }
};

// Polls up to N 16-byte lines until both words of each carry `tag`: line i
// (used where bit i of `mask` is set) is at base + (i / 2) * pair_stride +
// (i odd ? off1 : off0) words.  Every outstanding load is issued before any is
// checked, so the lines cost one round trip together rather than one each.
template <int N>
__device__ __forceinline__ void get_lines(const Poll& pl, const uint64_t* base, size_t pair_stride, size_t off0,
                                          size_t off1, uint32_t mask, uint32_t tag, uint2 (&out)[N]) {
  uint32_t pending = mask;
  uint64_t t0 = 0;
  for (unsigned it = 0; pending; ++it) {
    uint4 v[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((pending >> i) & 1u)
        asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                     : "l"(base + (size_t)(i >> 1) * pair_stride + ((i & 1) ? off1 : off0))
                     : "memory");
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((pending >> i) & 1u) {
        out[i] = make_uint2(v[i].x, v[i].z);
        if (v[i].y == tag && v[i].w == tag) pending &= ~(1u << i);
      }
    if (!pending) break;
    if (it == 0) t0 = gtimer();
    if ((it & 7u) == 7u && pl.stop(t0)) {
      pl.fail();
      break;
    }
  }
}

// The same with each line's address given.
template <int N>
__device__ __forceinline__ void get_lines_at(const Poll& pl, const uint64_t* const (&at)[N], uint32_t mask,
                                             uint32_t tag, uint2 (&out)[N]) {
  uint32_t pending = mask;
  uint64_t t0 = 0;
  for (unsigned it = 0; pending; ++it) {
    uint4 v[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((pending >> i) & 1u)
        asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                     : "l"(at[i])
                     : "memory");
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((pending >> i) & 1u) {
        out[i] = make_uint2(v[i].x, v[i].z);
        if (v[i].y == tag && v[i].w == tag) pending &= ~(1u << i);
      }
    if (!pending) break;
    if (it == 0) t0 = gtimer();
    if ((it & 7u) == 7u && pl.stop(t0)) {
      pl.fail();
      break;
    }
  }
}

__device__ __forceinline__ uint32_t bf2_bits(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t bf2_bits(bf16 lo, bf16 hi) {
  return (uint32_t)*reinterpret_cast<const uint16_t*>(&lo) |
         ((uint32_t)*reinterpret_cast<const uint16_t*>(&hi) << 16);
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

// c += A . B for one m16n8k16 tile with all four A registers given.
__device__ __forceinline__ void mma16816_a4(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ int phase_kind(int L, int ph) { return ph == 5 * L ? PH_HEAD : ph % 5; }

// Two warp sums with one reduction tree: lane 0 returns the sum of u over the
// warp, lane 16 the sum of v.  Each total is added up in the same order as
// warp_sum's butterfly (lane l with l ^ 16, then ^ 8, ^ 4, ^ 2, ^ 1), so the
// results are bitwise those of two warp_sum calls.
__device__ __forceinline__ float warp_sum_pair(float u, float v, int lane) {
  const bool hi = (lane & 16) != 0;
  float keep = hi ? v : u;
  keep += __shfl_xor_sync(0xffffffffu, hi ? u : v, 16);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
  return keep;
}

// The weight rows a CTA streams in one phase: rows [r0, r1) of w [N][K], in
// stages of rs whole rows.  Rows are dealt out in contiguous blocks of whole
// units: a RoPE pair for q/k/v (one tagged word of q, k or v), two rows for o
// and down (one word of x), two gate/up pairs for gate/up (one word of s).
// The o and down phases split their rows alike, so a CTA owns the same rows
// of the residual stream in both.
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
    case PH_O: o.w = (const bf16*)lw->wo; N = p.H; o.K = p.qd; unit = 2; break;
    case PH_GU: o.w = (const bf16*)lw->wgu; N = 2 * p.I; o.K = p.H; unit = 4; break;
    case PH_DOWN: o.w = (const bf16*)lw->wd; N = p.H; o.K = p.I; unit = 2; break;
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
  uint8_t* tiles = smem + sl::kTiles;
  uint8_t* ring = smem + sl::kRing;
  PLayer* layers = reinterpret_cast<PLayer*>(smem + Y.layers);
  float* yrow = reinterpret_cast<float*>(smem + sl::kYrow);
  float* part = reinterpret_cast<float*>(smem + sl::kPart);
  float* xres = reinterpret_cast<float*>(smem + sl::kXres);
  float* ebias = reinterpret_cast<float*>(smem + sl::kEbias);
  float2* ecs = reinterpret_cast<float2*>(smem + sl::kEcs);
  float* mlw = reinterpret_cast<float*>(smem + sl::kMlw);
  float* amv = reinterpret_cast<float*>(smem + sl::kAmv);
  long long* ami = reinterpret_cast<long long*>(smem + sl::kAmi);
  bf16* xbuf = reinterpret_cast<bf16*>(smem + sl::kXbuf);
  bf16* qst = reinterpret_cast<bf16*>(smem + sl::kQst);
  bf16* kvn = reinterpret_cast<bf16*>(smem + sl::kKvn);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Y.bars);
  uint64_t* empty = full + RING;
  uint64_t* abar = reinterpret_cast<uint64_t*>(smem + sl::kAbar);
  int* s_flags = reinterpret_cast<int*>(smem + sl::kFlags);  // [0] position, [1] step, [2] tiles pre-issued

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, bid = blockIdx.x;
  const int nph = p.run_head ? 5 * L + 1 : 5 * L;
  const uint64_t dl = p.deadline_ns;

  // the layer table in shared memory; the step's position and counter
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
    s_flags[0] = __ldcg(p.lens);
    s_flags[1] = (int)__ldcg(p.epoch);
    s_flags[2] = 0;
  }
  __syncthreads();
  const int pos = s_flags[0];  // the new token's position
  const int alen = pos + 1;    // keys attended (the new token included)
  // tag of phase ph's outputs in this step (unique per step and phase)
  const uint32_t tbase = (uint32_t)s_flags[1] * (uint32_t)(nph + 1) + 1u;
  auto wtag = [&](int ph) { return tbase + (uint32_t)ph; };
  // what a reader of phase ph's outputs waits for (the test hook makes one phase's
  // outputs unrecognisable to its readers)
  auto rtag = [&](int ph) { return wtag(ph) ^ (ph == p.stall_phase ? 0x80000000u : 0u); };

  // ================================================================ producer
  // One lane walks this CTA's stages of the whole step and issues one bulk
  // copy per stage as soon as its slot is free; a second cursor runs
  // l2_ahead stages in front and pulls them into L2.
  if (warp >= kCW) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == kCW && lane == 0) {
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
      long long gs = 0;
      for (; cur.valid(nph); ++gs) {
        if (gs >= RING && !bwait(&empty[slot], par ^ 1u, dl, p.sync)) {
          // the consumers stopped: issuing into a slot still in use would
          // break the ring's protocol, so stop here
          atomicOr(p.err, 2);
          atomicExch(p.sync, 1u);
          break;
        }
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
      // every copy issued has landed before the CTA may exit (these waits
      // only block if an earlier bounded wait gave up)
      for (int sl = 0; sl < RING; ++sl)
        if (gs > sl) bwait(&full[sl], (uint32_t)(((gs - 1 - sl) / RING) & 1), dl);
    }
    return;
  }

  // =============================================================== consumers
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
  const int ct = tid;
  const int Gq = p.nh / p.nkv;
  const int half = p.hd >> 1;
  const Poll pl{dl, p.sync, p.err};
  long long gs = 0;    // weight stages consumed
  int c_slot = 0;      // ring slot and parity of the next stage
  uint32_t c_par = 0;
  int ac = 0;          // attention tiles consumed
  float best_v = -INFINITY;  // lm_head: this warp's argmax over its rows
  long long best_i = LLONG_MAX;

  // The rows of the residual stream this CTA owns in the o and down phases,
  // kept here between its epilogues.
  {
    const int units = p.H / 2;
    const int r0 = (int)((long long)bid * units / G) * 2, r1 = (int)((long long)(bid + 1) * units / G) * 2;
    const bf16* src = reinterpret_cast<const bf16*>(p.x);
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
  // the phase's input vector into xbuf: from tagged words (bf16 pairs) ...
  auto stage_tagged = [&](const uint64_t* ll, int nwords, uint32_t tag) {
    uint2 got[2];
    uint32_t mask = 0;
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (ct + kCT * k < nwords / 2) mask |= 1u << k;
    get_lines<2>(pl, ll, 0, 2 * (size_t)ct, 2 * (size_t)(ct + kCT), mask, tag, got);
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if ((mask >> k) & 1u) reinterpret_cast<uint2*>(xbuf)[ct + kCT * k] = got[k];
    csync();
  };
  // ... or from plain bf16 memory
  auto stage_plain = [&](const bf16* src, int n) {
    for (int c = ct; c < n / 8; c += kCT) reinterpret_cast<uint4*>(xbuf)[c] = __ldcg(reinterpret_cast<const uint4*>(src) + c);
    csync();
  };
  // xr = this lane's pieces of xbuf, bf16(rmsnorm(xbuf) * nw) if nw is given,
  // as packed bf16 (every value is a bf16 either way): every warp normalises
  // the whole vector itself.
  auto input_regs = [&](bool norm, const uint4 (&nwr)[NCH], uint4 (&xr)[NCH]) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) xr[i] = reinterpret_cast<const uint4*>(xbuf)[lane + 32 * i];
    if (!norm) return;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      float f[8];
      unpack16<bf16>(xr[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)(NCH * 256) + p.eps);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      float f[8], wf[8];
      unpack16<bf16>(xr[i], f);
      unpack16<bf16>(nwr[i], wf);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = round_st<bf16>(f[e] * inv * wf[e]);
      xr[i] = pack16<bf16>(f);
    }
  };

  // The next stage of the ring: waits until it has landed, returns its slot.
  auto take_stage = [&]() {
    const int slot = c_slot;
    const uint32_t par = c_par;
    if (++c_slot == RING) {
      c_slot = 0;
      c_par ^= 1u;
    }
    ++gs;
    if (!bwait(&full[slot], par, dl, p.sync) && lane == 0) atomicOr(p.err, 2);
    return slot;
  };

  // The lm_head's stages, one at a time: warp w takes rows w, w + 8, ... of
  // each stage; the logits are written and the warp's argmax kept.
  auto consume_head = [&](const PW& pw, const uint4 (&xr)[NCH]) {
    for (int r = pw.r0; r < pw.r1; r += pw.rs) {
      const int s0 = take_stage();
      const int n = min(pw.rs, pw.r1 - r);
      const uint8_t* st = ring + (size_t)s0 * kSB;
      for (int rr = warp; rr < n; rr += kCW) {
        const uint4* wrow = reinterpret_cast<const uint4*>(st + (size_t)rr * pw.K * 2);
        float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          float wf[8], xf[8];
          unpack16<bf16>(wrow[lane + 32 * i], wf);
          unpack16<bf16>(xr[i], xf);
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e & 3] = fmaf(wf[e], xf[e], a[e & 3]);
        }
        const float y = warp_sum((a[0] + a[1]) + (a[2] + a[3]));
        const int row = r + rr;
        if (lane == 0) p.logits[row] = y;
        if (am_better(y, row, best_v, best_i)) {
          best_v = y;
          best_i = row;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s0]);
    }
  };

  // The stages of the other short-row phases, two at a time: warp w takes
  // rows w, w + 8, ... of each stage, row rr of both stages together, so that
  // the two rows' loads and products overlap and share one reduction tree;
  // the row results go to yrow.
  auto consume_short = [&](const PW& pw, const uint4 (&xr)[NCH]) {
    for (int r = pw.r0; r < pw.r1; r += 2 * pw.rs) {
      const bool two = r + pw.rs < pw.r1;
      const int s0 = take_stage();
      const int s1 = two ? take_stage() : s0;
      const int n0 = min(pw.rs, pw.r1 - r);
      const int n1 = two ? min(pw.rs, pw.r1 - r - pw.rs) : 0;
      const uint8_t* st0 = ring + (size_t)s0 * kSB;
      const uint8_t* st1 = ring + (size_t)s1 * kSB;
      for (int rr = warp; rr < n0; rr += kCW) {
        const bool has1 = rr < n1;  // warp-uniform
        const uint4* w0 = reinterpret_cast<const uint4*>(st0 + (size_t)rr * pw.K * 2);
        const uint4* w1 = reinterpret_cast<const uint4*>(st1 + (size_t)(has1 ? rr : 0) * pw.K * 2);
        float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          float wf[8], vf[8], xf[8];
          unpack16<bf16>(w0[lane + 32 * i], wf);
          unpack16<bf16>(has1 ? w1[lane + 32 * i] : make_uint4(0u, 0u, 0u, 0u), vf);
          unpack16<bf16>(xr[i], xf);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            a[e & 3] = fmaf(wf[e], xf[e], a[e & 3]);
            b[e & 3] = fmaf(vf[e], xf[e], b[e & 3]);
          }
        }
        // lane 0: row rr of the first stage, lane 16: of the second
        const float y = warp_sum_pair((a[0] + a[1]) + (a[2] + a[3]), (b[0] + b[1]) + (b[2] + b[3]), lane);
        if (lane == 0) yrow[r + rr - pw.r0] = y;
        if (lane == 16 && has1) yrow[r + pw.rs + rr - pw.r0] = y;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s0]);
        if (two) mbar_arrive(&empty[s1]);
      }
    }
  };

  // The stages of the down phase, two at a time: one row per stage, warp w
  // takes column pieces [w * cpw, (w + 1) * cpw) of both rows.
  auto consume_long = [&](const PW& pw, const float (&xf)[NQ][8]) {
    const int cpw = pw.K / 8 / kCW;
    for (int r = pw.r0; r < pw.r1; r += 2 * pw.rs) {
      const bool two = r + pw.rs < pw.r1;  // warp-uniform
      const int s0 = take_stage();
      const int s1 = two ? take_stage() : s0;
      const uint4* w0 = reinterpret_cast<const uint4*>(ring + (size_t)s0 * kSB) + warp * cpw;
      const uint4* w1 = reinterpret_cast<const uint4*>(ring + (size_t)s1 * kSB) + warp * cpw;
      float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        if (lane + 32 * q < cpw) {
          float wf[8], vf[8];
          unpack16<bf16>(w0[lane + 32 * q], wf);
          unpack16<bf16>(two ? w1[lane + 32 * q] : make_uint4(0u, 0u, 0u, 0u), vf);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            a[e & 3] = fmaf(wf[e], xf[q][e], a[e & 3]);
            b[e & 3] = fmaf(vf[e], xf[q][e], b[e & 3]);
          }
        }
      }
      // lane 0: the first stage's row, lane 16: the second's
      const float y = warp_sum_pair((a[0] + a[1]) + (a[2] + a[3]), (b[0] + b[1]) + (b[2] + b[3]), lane);
      if (lane == 0) part[warp * kDMax + (r - pw.r0)] = y;
      if (lane == 16 && two) part[warp * kDMax + (r + pw.rs - pw.r0)] = y;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s0]);
        if (two) mbar_arrive(&empty[s1]);
      }
    }
  };

  // ---- attention work items: (kv head, split) pairs, item = split * nkv + kv
  // head.  A split is a run of tiles of 64 keys: one tile per split while the
  // splits fit (at most nsplit per kv head, and the last nh CTAs are left to
  // the mergers), so a short context is spread one tile per CTA.
  struct AItem {
    int gq, split, ntiles, tps, t0, t1, nact;
  };
  auto attn_item = [&](int item) {
    AItem a;
    a.gq = item % p.nkv;
    a.split = item / p.nkv;
    a.ntiles = (alen + kAT - 1) / kAT;
    const int smax = max(1, min(p.nsplit, (G - p.nh) / p.nkv));
    const int active = min(smax, a.ntiles);
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
  // The first two tiles of this CTA's first attention item of layer l, issued
  // a layer ahead (at the start for layer 0, else when layer l - 1's
  // attention is done with the buffers) so that they land behind the weight
  // copies queued on this SM long before they are needed; the tile holding
  // the new position gets that row patched in later.
  auto prefetch_tiles = [&](int l) {
    if (ct != 0) return;
    s_flags[2] = 0;
    if (bid < aitems && l < L) {
      const AItem a = attn_item(bid);
      for (int q = 0; q < 2 && a.t0 + q < a.t1; ++q) {
        tile_issue(l, a.gq, a.t0 + q, ac + q);
        s_flags[2] = q + 1;
      }
    }
  };
  prefetch_tiles(0);

  for (int ph = 0; ph < nph; ++ph) {
    const int kind = phase_kind(L, ph);
    const int l = ph / 5;
    PW pw;
    phase_w(p, layers, ph, bid, G, pw);
    unsigned long long* ctr = p.ctrace ? p.ctrace + ((size_t)ph * G + bid) * 4 : nullptr;
    if (ctr && ct == 0) ctr[0] = gtimer();
    if (p.trace && ct == 0) {  // the phase's start (latest, and CTA 0's)
      const unsigned long long t = gtimer();
      atomicMax(&p.trace[ph * 4 + 3], t);
      if (bid == 0) p.trace[ph * 4 + 1] = t;
    }
    uint4 nwr[NCH];    // the RMSNorm weight pieces of this phase (loaded before its input)
    uint4 xr[NCH];     // short-row phases: this lane's pieces lane + 32 i of the input vector

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
    } else if (kind == PH_GU) {
      load_nw(layers[l].post_norm, nwr);
    } else if (kind == PH_HEAD) {
      load_nw(p.final_norm, nwr);
    }

    // ---- the phase's input, then its weight stages
    if (kind == PH_ATTN) {
      // Attention over the cache on the tensor cores with the keys on M.  Per
      // tile of 64 keys: S^T = K q^T (warp w: keys 16 (w % 4) .. + 15 against
      // the kv head's query heads on N, over head dims 64 (w / 4) .. + 63; the
      // two halves are added in shared memory), an online softmax per query
      // head (warp h takes head h: keys lane and lane + 32), then O^T += V^T P
      // (warp w: head dims 16 w .. + 15; P as bf16 high and low parts, so the
      // probabilities keep ~16 significant bits).  The split's partial
      // (unnormalised o, max, sum per query head) goes out from the
      // accumulators; CTA G - 1 - h merges the splits of query head h.
      const int g8 = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
      const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: lane addresses row mr of matrix mi
      const float sl2 = p.scale * kLog2e;
      const uint32_t tq = rtag(ph - 1), ta = wtag(ph);
      float* Sp = reinterpret_cast<float*>(xbuf);  // [2 dim halves][64 keys][8 heads], heads swizzled
      bf16* Ph = reinterpret_cast<bf16*>(yrow);     // [8 heads][kPS keys] P, high part
      bf16* Pl = Ph + kAGMax * kPS;                  // low part
      float* alph = mlw;                             // [8] this tile's rescale per head
      float* ew = mlw + kAGMax;                      // [kSplitMax + 1] merger: split weights, 1 / sum
      auto sp_at = [](int dh, int key, int h) { return (dh * kAT + key) * kAGMax + (h ^ ((key >> 2) & 7)); };
      const size_t hstride = kHD + 2;  // words per (split, head) partial
      for (int item = bid; item < aitems; item += G) {
        const AItem a = attn_item(item);
        if (a.t0 >= a.t1) continue;
        const int nt = a.t1 - a.t0;
        const bool last = a.t1 == a.ntiles;  // this split holds the new position
        const int pre = item == bid ? s_flags[2] : 0;
        if (ct == 0)
          for (int q = pre; q < 2 && q < nt; ++q) tile_issue(l, a.gq, a.t0 + q, ac + q);
        // q of the kv head's query heads (and the new K/V row), from the tagged words
        for (int v = ct; v < Gq * half / 2; v += kCT) {
          const int hh = v / (half / 2), j = 2 * (v % (half / 2));
          const uint2 d = pl.get2(p.ll.q + (size_t)(a.gq * Gq + hh) * half + j, tq);
          bf16* qh = qst + hh * kHD;
          qh[j] = __ushort_as_bfloat16((unsigned short)(d.x & 0xffffu));
          qh[j + half] = __ushort_as_bfloat16((unsigned short)(d.x >> 16));
          qh[j + 1] = __ushort_as_bfloat16((unsigned short)(d.y & 0xffffu));
          qh[j + 1 + half] = __ushort_as_bfloat16((unsigned short)(d.y >> 16));
        }
        if (last)
          for (int v = ct; v < half; v += kCT) {  // K pairs, then V pairs
            const int sel = v / (half / 2), j = 2 * (v % (half / 2));
            const uint2 d = pl.get2(p.ll.kv + (size_t)(sel * p.nkv + a.gq) * half + j, tq);
            bf16* r = kvn + sel * kHD;
            r[j] = __ushort_as_bfloat16((unsigned short)(d.x & 0xffffu));
            r[j + half] = __ushort_as_bfloat16((unsigned short)(d.x >> 16));
            r[j + 1] = __ushort_as_bfloat16((unsigned short)(d.y & 0xffffu));
            r[j + 1 + half] = __ushort_as_bfloat16((unsigned short)(d.y >> 16));
          }
        csync();
        if (ctr && ct == 0 && item == bid) ctr[1] = gtimer();  // attention: q and the new K/V row in
        const int kq = 16 * (warp & 3), dh = warp >> 2;
        // B fragments of q^T (head dims x query heads) for this warp's dim half;
        // heads past the group are zero
        uint32_t qb[4][2];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const bf16* qrow = qst + (g8 < Gq ? g8 : 0) * kHD + 64 * dh + 16 * ks + 2 * t4;
          qb[ks][0] = g8 < Gq ? *reinterpret_cast<const uint32_t*>(qrow) : 0u;
          qb[ks][1] = g8 < Gq ? *reinterpret_cast<const uint32_t*>(qrow + 8) : 0u;
        }
        // O^T accumulators: head dims 16 warp + g8 (+ 8) x heads 2 t4 (+ 1), from
        // the high and the low part of P
        float oh[4] = {0.f, 0.f, 0.f, 0.f}, ol[4] = {0.f, 0.f, 0.f, 0.f};
        float m_run = -INFINITY, l_run = 0.f;  // softmax of head `warp`
        for (int i = 0; i < nt; ++i) {
          const int li = ac + i, stg = li & 1;
          const int t = a.t0 + i;
          if (!bwait(&abar[stg], (uint32_t)((li >> 1) & 1), dl) && lane == 0) atomicOr(p.err, 2);
          uint8_t* tk = tiles + (size_t)stg * 2 * kTile;
          uint8_t* tv = tk + kTile;
          if (t == a.ntiles - 1) {
            // the tile holding the new position: its row comes from the
            // published K/V (the cache row may have been read before it
            // existed), and the rows after it are stale cache rows (possibly not
            // finite: their scores are masked, their V rows zeroed)
            const int r = pos - t * kAT;
            if (warp == 0) {
              const int c = lane & 15;
              uint8_t* dst = (lane < 16 ? tk : tv) + (c >> 3) * 8192 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
              *reinterpret_cast<uint4*>(dst) = reinterpret_cast<const uint4*>(kvn + (lane < 16 ? 0 : kHD))[c];
            }
            for (int c = ct; c < (kAT - 1 - r) * 16; c += kCT) {
              const int vr = r + 1 + c / 16, ch = c % 16;
              *reinterpret_cast<uint4*>(tv + (ch >> 3) * 8192 + vr * 128 + (((ch & 7) ^ (vr & 7)) << 4)) =
                  make_uint4(0u, 0u, 0u, 0u);
            }
            csync();
          }
          const uint32_t ka = smem_u32(tk), va = smem_u32(tv);
          // ---- S^T, keys kq .. kq + 15 x heads, over this warp's dim half
          {
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4(ka + (uint32_t)(dh * 8192) + swz_off(kq + mr + ((mi & 1) << 3), 16 * ks + ((mi >> 1) << 3)),
                      r0, r1, r2, r3);
              mma16816_a4((ks & 1) ? sb : sa, r0, r1, r2, r3, qb[ks][0], qb[ks][1]);
            }
            Sp[sp_at(dh, kq + g8, 2 * t4)] = sa[0] + sb[0];
            Sp[sp_at(dh, kq + g8, 2 * t4 + 1)] = sa[1] + sb[1];
            Sp[sp_at(dh, kq + g8 + 8, 2 * t4)] = sa[2] + sb[2];
            Sp[sp_at(dh, kq + g8 + 8, 2 * t4 + 1)] = sa[3] + sb[3];
          }
          csync();
          // ---- online softmax of head `warp` over the tile's keys lane, lane + 32
          {
            const int h = warp;
            bf16* ph = Ph + h * kPS;
            bf16* plo = Pl + h * kPS;
            if (h < Gq) {
              const int kb = t * kAT;
              float s0 = (Sp[sp_at(0, lane, h)] + Sp[sp_at(1, lane, h)]) * sl2;
              float s1 = (Sp[sp_at(0, lane + 32, h)] + Sp[sp_at(1, lane + 32, h)]) * sl2;
              if (kb + lane >= alen) s0 = -INFINITY;
              if (kb + lane + 32 >= alen) s1 = -INFINITY;
              // key kb is always visible, so the tile's max is finite
              const float mnew = fmaxf(m_run, warp_max(fmaxf(s0, s1)));
              const float alpha = exp2f(m_run - mnew);  // 0 on the first tile
              const float p0 = exp2f(s0 - mnew), p1 = exp2f(s1 - mnew);
              l_run = l_run * alpha + warp_sum(p0 + p1);
              m_run = mnew;
              const bf16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
              ph[lane] = h0;
              ph[lane + 32] = h1;
              plo[lane] = __float2bfloat16_rn(p0 - __bfloat162float(h0));
              plo[lane + 32] = __float2bfloat16_rn(p1 - __bfloat162float(h1));
              if (lane == 0) alph[h] = alpha;
            } else {  // no such head: zero P
              const bf16 z = __float2bfloat16_rn(0.f);
              ph[lane] = ph[lane + 32] = plo[lane] = plo[lane + 32] = z;
              if (lane == 0) alph[h] = 1.f;
            }
          }
          csync();
          // ---- O^T += V^T P for head dims 16 warp .. + 15
          {
            const float a0 = alph[2 * t4], a1 = alph[2 * t4 + 1];
            oh[0] *= a0;
            oh[1] *= a1;
            oh[2] *= a0;
            oh[3] *= a1;
            ol[0] *= a0;
            ol[1] *= a1;
            ol[2] *= a0;
            ol[3] *= a1;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4_t(va + (uint32_t)((warp >> 2) * 8192) +
                            swz_off(16 * ks + mr + ((mi >> 1) << 3), 16 * (warp & 3) + ((mi & 1) << 3)),
                        r0, r1, r2, r3);
              const int kk = g8 * kPS + 16 * ks + 2 * t4;
              mma16816_a4(oh, r0, r1, r2, r3, *reinterpret_cast<const uint32_t*>(Ph + kk),
                          *reinterpret_cast<const uint32_t*>(Ph + kk + 8));
              mma16816_a4(ol, r0, r1, r2, r3, *reinterpret_cast<const uint32_t*>(Pl + kk),
                          *reinterpret_cast<const uint32_t*>(Pl + kk + 8));
            }
          }
          if (i + 2 < nt) {
            csync();  // every warp is done with this stage
            if (ct == 0) tile_issue(l, a.gq, t + 2, li + 2);
          }
        }
        ac += nt;
        if (ctr && ct == 0 && item == bid) ctr[2] = gtimer();  // attention: tiles done
        // ---- this split's partial, from the accumulators
        uint64_t* pb = p.ll.part + (size_t)(a.gq * kSplitMax + a.split) * Gq * hstride;
        const int d0 = 16 * warp + g8;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hh = 2 * t4 + e;
          if (hh < Gq) {
            ll_put(pb + hh * hstride + d0, __float_as_uint(oh[e] + ol[e]), ta);
            ll_put(pb + hh * hstride + d0 + 8, __float_as_uint(oh[2 + e] + ol[2 + e]), ta);
          }
        }
        if (warp < Gq && lane == 0)
          ll_put2(pb + warp * hstride + kHD, __float_as_uint(m_run), __float_as_uint(l_run), ta);
        csync();  // the next item's q, scores and P overwrite this one's
      }
      // ---- the merge of query head mh = G - 1 - bid over its splits:
      // o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.  The
      // partials are staged in the tile buffers (free: every tile this CTA
      // issued has been waited on and read).
      const int mh = G - 1 - bid;
      if (mh >= 0 && mh < p.nh) {
        const AItem a = attn_item(0);
        const int gq = mh / Gq, hh = mh % Gq;
        const int lps = (int)(hstride / 2);  // 16-byte lines per split partial
        const int nlines = a.nact * lps;
        float* pst = reinterpret_cast<float*>(tiles);  // [nact][hstride]
        const uint64_t* pb0 = p.ll.part + (size_t)gq * kSplitMax * Gq * hstride + (size_t)hh * hstride;
        for (int l0 = 0; l0 < nlines; l0 += 4 * kCT) {
          const uint64_t* at[4];
          uint32_t mask = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int L = l0 + ct + kCT * k;
            at[k] = pb0;
            if (L < nlines) {
              mask |= 1u << k;
              at[k] = pb0 + (size_t)(L / lps) * Gq * hstride + 2 * (L % lps);
            }
          }
          uint2 got[4];
          get_lines_at<4>(pl, at, mask, rtag(ph), got);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if ((mask >> k) & 1u) reinterpret_cast<uint2*>(pst)[l0 + ct + kCT * k] = got[k];
        }
        csync();
        if (warp == 0) {
          float M = -INFINITY;
          for (int sp = lane; sp < a.nact; sp += 32) M = fmaxf(M, pst[sp * hstride + kHD]);
          M = warp_max(M);
          float Ls = 0.f;
          for (int sp = lane; sp < a.nact; sp += 32) {
            const float e = exp2f(pst[sp * hstride + kHD] - M);
            ew[sp] = e;
            Ls = fmaf(e, pst[sp * hstride + kHD + 1], Ls);
          }
          Ls = warp_sum(Ls);
          if (lane == 0) ew[kSplitMax] = Ls > 0.f ? 1.f / Ls : 0.f;
        }
        csync();
        if (ct < half) {
          float o0 = 0.f, o1 = 0.f;
          for (int sp = 0; sp < a.nact; ++sp) {
            o0 = fmaf(ew[sp], pst[sp * hstride + 2 * ct], o0);
            o1 = fmaf(ew[sp], pst[sp * hstride + 2 * ct + 1], o1);
          }
          const float inv = ew[kSplitMax];
          ll_put(p.ll.att + (size_t)mh * half + ct, bf2_bits(o0 * inv, o1 * inv), ta);
        }
      }
      fence_proxy_async_smem();  // the tile buffers are TMA destinations again
      csync();
      prefetch_tiles(l + 1);
    } else if (kind == PH_DOWN) {
      uint4 xs[NQ];  // this lane's pieces of the warp's column slice of s (bf16), then as fp32
      float xf[NQ][8];
      const int cpw = pw.K / 8 / kCW;
      {
        const uint64_t* sbase = p.ll.s + (size_t)(warp * cpw + lane) * 4;
        constexpr int QH = (NQ + 1) / 2;  // pieces polled per batch
#pragma unroll
        for (int q0 = 0; q0 < NQ; q0 += QH) {
          uint2 got[2 * QH];
          uint32_t mask = 0;
#pragma unroll
          for (int q = 0; q < QH; ++q)
            if (q0 + q < NQ && lane + 32 * (q0 + q) < cpw) mask |= 3u << (2 * q);
          get_lines<2 * QH>(pl, sbase + (size_t)(32 * q0) * 4, 32 * 4, 0, 2, mask, rtag(ph - 1), got);
#pragma unroll
          for (int q = 0; q < QH; ++q)
            if (q0 + q < NQ)
              xs[q0 + q] = (mask >> (2 * q)) & 1u
                               ? make_uint4(got[2 * q].x, got[2 * q].y, got[2 * q + 1].x, got[2 * q + 1].y)
                               : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (ctr && ct == 0) ctr[1] = gtimer();
#pragma unroll
      for (int q = 0; q < NQ; ++q) unpack16<bf16>(xs[q], xf[q]);
      consume_long(pw, xf);
    } else {  // the short-row phases: q/k/v, o, gate/up, lm_head
      if (kind == PH_QKV && l == 0) {
        // layer 0: the embedding row (an id outside the vocabulary sets bit 0 of
        // the error word and reads row 0), or the caller's input
        const bf16* src = reinterpret_cast<const bf16*>(p.x);
        if (p.embed_in) {
          long long id = __ldcg(p.ids);
          if (id < 0 || id >= p.V) {
            if (ct == 0 && bid == 0) atomicOr(p.err, 1);
            id = 0;
          }
          src = reinterpret_cast<const bf16*>(p.embed) + (size_t)id * p.H;
        }
        stage_plain(src, p.H);
      } else if (kind == PH_O) {
        stage_tagged(p.ll.att, p.qd / 2, rtag(ph - 1));
      } else {  // x from the previous o or down phase
        stage_tagged(p.ll.x, p.H / 2, rtag(ph - 1));
      }
      if (ctr && ct == 0) ctr[1] = gtimer();
      input_regs(kind != PH_O, nwr, xr);
      if (kind == PH_HEAD)
        consume_head(pw, xr);
      else
        consume_short(pw, xr);
    }

    // ---- phase epilogue from the parked row results and staged operands
    csync();
    if (ctr && ct == 0 && kind != PH_ATTN) ctr[2] = gtimer();
    const uint32_t tw = wtag(ph);
    if (kind == PH_QKV) {
      const size_t loff = (size_t)l * p.kv_layer_stride;
      for (int i = ct; 2 * i < pw.r1 - pw.r0; i += kCT) {
        const int n = pw.r0 + 2 * i;
        const int hs = n / p.hd, j = (n % p.hd) >> 1;
        const float va = round_st<bf16>(yrow[2 * i] + ebias[2 * i]);
        const float vb = round_st<bf16>(yrow[2 * i + 1] + ebias[2 * i + 1]);
        bf16 ra, rb;
        if (hs < p.nh + p.nkv) {
          const float2 cs = ecs[i];
          ra = __float2bfloat16_rn(va * cs.x - vb * cs.y);
          rb = __float2bfloat16_rn(vb * cs.x + va * cs.y);
        } else {
          ra = __float2bfloat16_rn(va);
          rb = __float2bfloat16_rn(vb);
        }
        if (hs < p.nh) {
          ll_put(p.ll.q + (size_t)hs * half + j, bf2_bits(ra, rb), tw);
        } else {
          const int kvh = hs - p.nh;  // 0 .. nkv - 1: K heads, nkv .. 2 nkv - 1: V heads
          bf16* dst = reinterpret_cast<bf16*>(kvh < p.nkv ? p.kc : p.vc) + loff +
                      ((size_t)(kvh % p.nkv) * p.max_seq + pos) * p.hd;
          dst[j] = ra;
          dst[j + half] = rb;
          ll_put(p.ll.kv + (size_t)kvh * half + j, bf2_bits(ra, rb), tw);
        }
      }
    } else if (kind == PH_O || kind == PH_DOWN) {
      bf16* xw = reinterpret_cast<bf16*>(p.x);
      for (int i = ct; 2 * i < pw.r1 - pw.r0; i += kCT) {
        float y0, y1;
        if (kind == PH_O) {
          y0 = yrow[2 * i];
          y1 = yrow[2 * i + 1];
        } else {
          y0 = y1 = 0.f;
#pragma unroll
          for (int w = 0; w < kCW; ++w) {
            y0 += part[w * kDMax + 2 * i];
            y1 += part[w * kDMax + 2 * i + 1];
          }
        }
        const bf16 x0 = __float2bfloat16_rn(xres[2 * i] + round_st<bf16>(y0));
        const bf16 x1 = __float2bfloat16_rn(xres[2 * i + 1] + round_st<bf16>(y1));
        const int n = pw.r0 + 2 * i;
        xw[n] = x0;
        xw[n + 1] = x1;
        xres[2 * i] = __bfloat162float(x0);
        xres[2 * i + 1] = __bfloat162float(x1);
        ll_put(p.ll.x + n / 2, bf2_bits(x0, x1), tw);
      }
    } else if (kind == PH_GU) {
      for (int i = ct; 4 * i < pw.r1 - pw.r0; i += kCT) {
        const float s0 = silu_mul(round_st<bf16>(yrow[4 * i]), round_st<bf16>(yrow[4 * i + 1]));
        const float s1 = silu_mul(round_st<bf16>(yrow[4 * i + 2]), round_st<bf16>(yrow[4 * i + 3]));
        ll_put(p.ll.s + pw.r0 / 4 + i, bf2_bits(s0, s1), tw);
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
        ll_put2(p.ll.am + 2 * bid, __float_as_uint(bv), (uint32_t)bi, tw);
      }
    }
    if (ct == 0) {
      if (ctr) ctr[3] = gtimer();
      if (p.trace) {
        const unsigned long long t = gtimer();
        atomicMax(&p.trace[ph * 4 + 0], t);
        if (bid == 0) p.trace[ph * 4 + 2] = t;
      }
    }
  }

  // ---- drain: every attention tile this CTA issued has landed before it
  // exits (the producer drains the weight ring)
  if (ct == 0) {
    for (int st = 0; st < 2; ++st)
      if (ac > st) bwait(&abar[st], (uint32_t)(((ac - 1 - st) / 2) & 1), dl);
  }

  // ---- CTA 0 wraps up the step: the token (argmax over the CTAs' partials,
  // which the order of the pairs alone decides), the length, the step counter
  if (bid == 0) {
    if (p.run_head) {
      float bv = -INFINITY;
      long long bi = LLONG_MAX;
      for (int c = ct; c < G; c += kCT) {
        const uint2 d = pl.get2(p.ll.am + 2 * c, rtag(nph - 1));
        if (am_better(__uint_as_float(d.x), (long long)d.y, bv, bi)) {
          bv = __uint_as_float(d.x);
          bi = (long long)d.y;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const long long oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (am_better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      csync();  // amv / ami are free again
      if (lane == 0) {
        amv[warp] = bv;
        ami[warp] = bi;
      }
      csync();
      if (ct == 0) {
        for (int w = 0; w < kCW; ++w)
          if (am_better(amv[w], ami[w], bv, bi)) {
            bv = amv[w];
            bi = ami[w];
          }
        p.next[0] = bi;
      }
    }
    if (ct == 0) {
      p.lens[0] += 1;
      *p.epoch += 1u;
    }
  }
}

// ======================================================================
namespace {
constexpr int kNCH = 6;  // H = 1536
constexpr int kNQ = 5;   // ceil(I / 8 / kCW / 32) for I = 8960

// the tagged buffers, each starting on a 16-byte boundary
struct LLSizes {
  size_t x, q, kv, att, s, part, am;
};
LLSizes ll_sizes(int H, int I, int nh, int nkv, int hd, int grid) {
  auto even = [](size_t n) { return (n + 1) / 2 * 2; };
  LLSizes z;
  z.x = even((size_t)H / 2);
  z.q = even((size_t)nh * hd / 2);
  z.kv = even((size_t)2 * nkv * hd / 2);
  z.att = even((size_t)nh * hd / 2);
  z.s = even((size_t)I / 2);
  z.part = even((size_t)nkv * kSplitMax * (nh / nkv) * (hd + 2));
  z.am = (size_t)2 * grid;
  return z;
}
}  // namespace

size_t sdecode_ll_words(int H, int I, int nh, int nkv, int hd, int grid) {
  const LLSizes z = ll_sizes(H, I, nh, nkv, hd, grid);
  return z.x + z.q + z.kv + z.att + z.s + z.part + z.am;
}

SDecodeLL sdecode_ll_carve(uint64_t* base, int H, int I, int nh, int nkv, int hd, int grid) {
  const LLSizes z = ll_sizes(H, I, nh, nkv, hd, grid);
  SDecodeLL b;
  b.x = base;
  b.q = b.x + z.x;
  b.kv = b.q + z.q;
  b.att = b.kv + z.kv;
  b.s = b.att + z.att;
  b.part = b.s + z.s;
  b.am = b.part + z.part;
  return b;
}

bool sdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd) {
  if (hd != kHD || nkv <= 0 || nh % nkv != 0 || nh / nkv > kAGMax || V <= 0) return false;
  if (H != kNCH * 256 || qd != H || H > kHMax || qkvd % 2 != 0) return false;
  if (I % (8 * kCW) != 0 || (I / 8 / kCW + 31) / 32 != kNQ || I * 2 > kSB || I * 2 <= kSB / 2)
    return false;
  return true;
}

size_t sdecode_sync_words() { return 4; }

int sdecode_max_ring(int L) {
  for (int ring = 8; ring >= 2; --ring)
    if (slayout(ring, L).total <= kSmemMax) return ring;
  return 0;
}

q2_status launch_sdecode(const SDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t st) {
  if (!sdecode_supported(p.H, p.I, p.V, p.nh, p.nkv, p.hd, p.qkvd, p.qd) || p.nsplit < 1 ||
      p.nsplit > kSplitMax || p.ring < 2 || p.L < 1) {
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
  const long long gu_rows = (long long)(2 * p.I / 4 + G - 1) / G * 4;
  const long long o_rows = (long long)(p.H / 2 + G - 1) / G * 2;
  if (qkv_rows > kQMax || gu_rows > kYMax || o_rows > kYMax || o_rows > kDMax) {
    set_error("streaming decode: too many rows per CTA for this device");
    return Q2_ERR_SHAPE;
  }
  if (G < p.nh + p.nkv) {  // a merger CTA per query head, and an attention CTA per kv head besides
    set_error("streaming decode: fewer SMs than query plus kv heads");
    return Q2_ERR_SHAPE;
  }
  auto kern = sdecode_kernel<kNCH, kNQ>;
  // The warpgroups' register split assumes exactly kLaunchRegs per thread at
  // launch; with any other count the split could not be honoured.
  cudaFuncAttributes fa;
  Q2_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
  if (fa.numRegs != kLaunchRegs) {
    set_error("streaming decode: the kernel was built with " + std::to_string(fa.numRegs) +
              " registers per thread, its register split assumes " + std::to_string(kLaunchRegs));
    return Q2_ERR_CUDA;
  }
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
