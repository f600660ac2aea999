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
constexpr int kThreads = (kC + 1) * 32;     // + one producer warp
constexpr int kSlot = 24 * 1024;            // ring slot (largest weight stage)
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
  size_t o_ring, o_act, o_qs, o_S, o_ml, o_red, o_ami, o_amv, o_bars, o_flag, total;
};

__host__ __device__ inline size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

PGeo make_geo(int mt, int act_elems) {
  PGeo g;
  g.act_elems = act_elems;
  size_t o = 2 * 2 * (size_t)kTileBytes;  // attention K/V tiles, two stages (reused by the O prologue)
  g.o_ring = o;                           // ring follows (filled below)
  size_t fixed = up((size_t)mt * act_elems * 2, 16) + kAGMax * kHD * 4 + kAGMax * kAT * 4 +
                 3 * kAGMax * 4 + kC * 4 * 4 + kC * 4 * 8 + kC * 4 * 4 + 64 * 8 + 64;
  long long room = (long long)kSmemMax - 1024 - (long long)o - (long long)fixed;
  int ring = (int)(room / kSlot);
  if (ring > 8) ring = 8;
  g.ring = ring;
  o += (size_t)ring * kSlot;
  g.o_act = o;
  o = up(o + (size_t)mt * act_elems * 2, 16);
  g.o_qs = o;
  o += kAGMax * kHD * 4;
  g.o_S = o;
  o += kAGMax * kAT * 4;
  g.o_ml = o;
  o += 3 * kAGMax * 4;
  g.o_red = o;
  o += kC * 4 * 4;
  g.o_ami = up(o, 8);
  o = g.o_ami + kC * 4 * 8;
  g.o_amv = o;
  o += kC * 4 * 4;
  g.o_bars = up(o, 8);
  o = g.o_bars + ((size_t)ring + 2) * 8 + (size_t)ring * 4;  // full[ring], abar[2], released[ring]
  o = up(o, 8);
  g.o_flag = o;
  o += 16;
  g.total = o + 1024;  // slack for aligning the base
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

// mbarrier wait with a deadline; false if it ran out.
__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (;;) {
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (gtimer() - t0 > kDeadlineNs) return false;
  }
}

// Wait until a shared-memory counter reaches `target` (deadline-bounded).
__device__ __forceinline__ bool wait_count(const unsigned* c, unsigned target) {
  const volatile unsigned* vc = c;
  if (*vc >= target) return true;
  const uint64_t t0 = gtimer();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (*vc >= target) return true;
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

__device__ __forceinline__ int swz(int r, int c) {
  return r * 128 + ((((c >> 3) ^ (r & 7)) << 4) | ((c & 7) << 1));
}

enum { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_GU = 3, PH_DOWN = 4, PH_HEAD = 5 };

struct WPhase {
  const bf16* w;
  int N, K, R, rpu, kind;
};

__device__ __forceinline__ int phase_kind(const PDecode& p, int ph) {
  return ph == 5 * p.L ? PH_HEAD : ph % 5;
}

__device__ __forceinline__ bool weight_phase(const PDecode& p, int ph, WPhase& wp) {
  const int kind = phase_kind(p, ph);
  if (kind == PH_ATTN) return false;
  const PLayer* Lw = kind == PH_HEAD ? nullptr : &p.layers[ph / 5];
  switch (kind) {
    case PH_QKV: wp.w = (const bf16*)Lw->wqkv; wp.N = p.qkvd; wp.K = p.H; wp.rpu = 2; break;
    case PH_O: wp.w = (const bf16*)Lw->wo; wp.N = p.H; wp.K = p.qd; wp.rpu = 1; break;
    case PH_GU: wp.w = (const bf16*)Lw->wgu; wp.N = 2 * p.I; wp.K = p.H; wp.rpu = 2; break;
    case PH_DOWN: wp.w = (const bf16*)Lw->wd; wp.N = p.H; wp.K = p.I; wp.rpu = 1; break;
    default: wp.w = (const bf16*)p.lm_head; wp.N = p.V; wp.K = p.H; wp.rpu = 1; break;
  }
  int r = 8;
  while (r > wp.rpu && r * wp.K * 2 > kSlot) r >>= 1;
  wp.R = r;
  wp.kind = kind;
  return true;
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
  long long* ami = reinterpret_cast<long long*>(smem + g.o_ami);
  float* amv = reinterpret_cast<float*>(smem + g.o_amv);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + g.o_bars);
  uint64_t* abar = full + g.ring;
  // released[slot]: cumulative count of consumer releases of that slot, kC per
  // use.  A cumulative count (rather than a parity wait on an mbarrier) lets a
  // consumer that runs several uses ahead of another warp tell exactly which
  // use of the slot is resident.
  unsigned* released = reinterpret_cast<unsigned*>(abar + 2);
  int* s_flags = reinterpret_cast<int*>(smem + g.o_flag);
  int& s_flag = s_flags[0];
  int& s_last_merge = s_flags[1];
  int& s_pre = s_flags[2];  // attention tiles of this CTA's first item already in flight

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, bid = blockIdx.x;
  const int nph = p.run_head ? 5 * p.L + 1 : 5 * p.L;
  const int RING = g.ring;

  if (tid == 0) {
    for (int i = 0; i < RING; ++i) {
      mbar_init(&full[i], 1);
      released[i] = 0;
    }
    mbar_init(&abar[0], 1);
    mbar_init(&abar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ================================================================ producer
  if (warp == kC) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      long long gs = 0;
      for (int ph = 0; ph < nph; ++ph) {
        WPhase wp;
        if (!weight_phase(p, ph, wp)) continue;
        const int Sn = (wp.N + wp.R - 1) / wp.R;
        const int sb = (int)((long long)bid * Sn / G), se = (int)((long long)(bid + 1) * Sn / G);
        for (int s = sb; s < se; ++s, ++gs) {
          const int slot = (int)(gs % RING);
          const long long k = gs / RING;
          // Reuse of a slot waits for every consumer release of its previous
          // use (their reads of the slot are complete before they release it).
          if (k >= 1 && !wait_count(&released[slot], (unsigned)(k * kC))) atomicOr(p.err, 2);
          const int rows = min(wp.R, wp.N - s * wp.R);
          const uint32_t bytes = (uint32_t)rows * wp.K * 2;
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_g2s_evict_first(ring + (size_t)slot * kSlot, wp.w + (size_t)s * wp.R * wp.K, bytes,
                               &full[slot], pol);
        }
      }
    }
    return;
  }

  // =============================================================== consumers
  const int ct = tid;
  const int G_q = p.nh / p.nkv;
  long long gs = 0;  // weight stages consumed so far (same sequence as the producer's)
  int ac = 0;        // attention tile loads issued so far
  const bf16* X = reinterpret_cast<const bf16*>(p.x);
  // Sequence lengths only change at the very end of the step: lane m keeps
  // token m's position.
  const int my_pos = lane < p.B ? p.lens[lane] : 0;
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
  float best_v = -INFINITY;
  long long best_i = LLONG_MAX;

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
          *reinterpret_cast<uint4*>(act + (size_t)m * K + k) = pack16<bf16>(f);
        }
      }
    }
    csync();
  };

  // One weight phase: stream this CTA's stages, run the epilogue per unit.
  auto gemv_phase = [&](const WPhase& wp, int l) {
    const int Sn = (wp.N + wp.R - 1) / wp.R;
    const int sb = (int)((long long)bid * Sn / G), se = (int)((long long)(bid + 1) * Sn / G);
    const int ns = se - sb;
    const int units = wp.R / wp.rpu;
    const uint32_t arrive_cnt = (uint32_t)(kC / units);
    const int K = wp.K, nch = K / 8;
    // MT == 1 and K == 1536: the activation stays in registers (6 chunks per lane).
    constexpr int NXR = MT == 1 ? 6 : 1;
    const bool regs = (MT == 1) && (K == 6 * 256);
    float xr[NXR][8];
    if (regs) {
#pragma unroll
      for (int i = 0; i < NXR; ++i) unpack16<bf16>(reinterpret_cast<const uint4*>(act)[lane + 32 * i], xr[i]);
    }
    for (int item = warp; item < ns * units; item += kC) {
      const int ls_ = item / units, u = item % units;
      const long long gsi = gs + ls_;
      const int slot = (int)(gsi % RING);
      const long long k = gsi / RING;
      // Every earlier use of the slot is released (so use k is the one the
      // producer fills next, and the full barrier's parity is unambiguous).
      if (k >= 1 && !wait_count(&released[slot], (unsigned)(k * kC)) && lane == 0) atomicOr(p.err, 2);
      if (!mwait(&full[slot], (uint32_t)(k & 1)) && lane == 0) atomicOr(p.err, 2);
      const uint8_t* stg = ring + (size_t)slot * kSlot;
      const int s = sb + ls_;
      const int row0 = s * wp.R;
      const int rows = min(wp.R, wp.N - row0);
      // Operands of the epilogue, loaded before the dot product so that their
      // latency overlaps it (lane m < B works for token m).
      const int n0e = row0 + u * wp.rpu;
      float e_b0 = 0.f, e_b1 = 0.f, e_x = 0.f;
      float2 e_cs = make_float2(1.f, 0.f);
      if (lane < p.B && n0e < wp.N) {
        if (wp.kind == PH_QKV) {
          const bf16* bias = reinterpret_cast<const bf16*>(p.layers[l].bqkv);
          e_b0 = to_f(bias[n0e]);
          e_b1 = to_f(bias[n0e + 1]);
          const int hs = n0e / p.hd;
          if (hs < p.nh + p.nkv) e_cs = p.rope[(size_t)my_pos * (p.hd >> 1) + ((n0e % p.hd) >> 1)];
        } else if (wp.kind == PH_O || wp.kind == PH_DOWN) {
          e_x = __bfloat162float(
              __ldcg(reinterpret_cast<const __nv_bfloat16*>(p.x) + (size_t)lane * p.H + n0e));
        }
      }
      float y[2][MT];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) y[r][m] = 0.f;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r >= wp.rpu) break;
        const int rr = u * wp.rpu + r;
        if (rr >= rows) break;
        const uint4* wrow = reinterpret_cast<const uint4*>(stg + (size_t)rr * K * 2);
        if (regs) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int i = 0; i < NXR; ++i) {
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
              if (m < p.B) {
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
      if (lane == 0) {
        __threadfence_block();
        atomicAdd(&released[slot], arrive_cnt);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) y[r][m] = warp_sum(y[r][m]);

      const int m = lane;
      if (m < p.B && m < MT) {
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int mm = 0; mm < MT; ++mm)
          if (mm == m) {
            y0 = y[0][mm];
            y1 = y[1][mm];
          }
        const int n0 = n0e;
        if (wp.kind == PH_O || wp.kind == PH_DOWN) {
          if (n0 < wp.N)
            reinterpret_cast<bf16*>(p.x)[(size_t)m * p.H + n0] = from_f<bf16>(e_x + round_st<bf16>(y0));
        } else if (wp.kind == PH_GU) {
          if (n0 + 1 < wp.N) {
            const float gv = round_st<bf16>(y0), uv = round_st<bf16>(y1);
            reinterpret_cast<bf16*>(p.s)[(size_t)m * p.I + (n0 >> 1)] = from_f<bf16>(silu_mul(gv, uv));
          }
        } else if (wp.kind == PH_QKV) {
          if (n0 + 1 < wp.N) {
            const int hs = n0 / p.hd, j = (n0 % p.hd) >> 1, half = p.hd >> 1;
            const float va = round_st<bf16>(y0 + e_b0);
            const float vb = round_st<bf16>(y1 + e_b1);
            const int pos = my_pos;
            const size_t loff = (size_t)l * p.kv_layer_stride + (size_t)m * p.kv_seq_stride;
            if (hs < p.nh + p.nkv) {
              const bf16 ra = from_f<bf16>(va * e_cs.x - vb * e_cs.y);
              const bf16 rb = from_f<bf16>(vb * e_cs.x + va * e_cs.y);
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
          if (n0 < wp.N) {
            p.logits[(size_t)m * p.V + n0] = y0;
            if (am_better(y0, n0, best_v, best_i)) {
              best_v = y0;
              best_i = n0;
            }
          }
        }
      }
    }
    gs += ns;
  };

  for (int ph = 0; ph < nph; ++ph) {
    const int kind = phase_kind(p, ph);
    const int l = ph / 5;
    // ---- wait until every CTA finished the previous phase
    if (ph > 0) {
      if (ct == 0) {
        const uint64_t t0 = gtimer();
        while (ld_acquire(&p.sync[ph - 1]) < (unsigned)G) {
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
      norm_prologue(rows_, reinterpret_cast<const bf16*>(p.layers[l].in_norm), p.H);
      WPhase wp;
      weight_phase(p, ph, wp);
      gemv_phase(wp, l);
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
      const bf16* A = reinterpret_cast<const bf16*>(p.att);
      for (int k = ct * 8; k < p.qd; k += kC * 32 * 8)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < p.B)
            *reinterpret_cast<uint4*>(act + (size_t)m * p.qd + k) =
                __ldcg(reinterpret_cast<const uint4*>(A + (size_t)m * p.qd + k));
      csync();
      WPhase wp;
      weight_phase(p, ph, wp);
      gemv_phase(wp, l);
    } else if (kind == PH_GU) {
      const bf16* rows_[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) rows_[m] = X + (size_t)m * p.H;
      norm_prologue(rows_, reinterpret_cast<const bf16*>(p.layers[l].post_norm), p.H);
      WPhase wp;
      weight_phase(p, ph, wp);
      gemv_phase(wp, l);
    } else if (kind == PH_DOWN) {
      const bf16* Sv = reinterpret_cast<const bf16*>(p.s);
      for (int k = ct * 8; k < p.I; k += kC * 32 * 8)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < p.B)
            *reinterpret_cast<uint4*>(act + (size_t)m * p.I + k) =
                __ldcg(reinterpret_cast<const uint4*>(Sv + (size_t)m * p.I + k));
      csync();
      WPhase wp;
      weight_phase(p, ph, wp);
      gemv_phase(wp, l);
    } else {  // PH_HEAD
      const bf16* rows_[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) rows_[m] = X + (size_t)m * p.H;
      norm_prologue(rows_, reinterpret_cast<const bf16*>(p.final_norm), p.H);
      WPhase wp;
      weight_phase(p, ph, wp);
      gemv_phase(wp, l);
      // this CTA's argmax partial per token
      if (lane < MT) {
        ami[warp * 4 + lane] = best_i;
        amv[warp * 4 + lane] = best_v;
      }
      csync();
      if (ct < p.B) {
        float bv = -INFINITY;
        long long bi = LLONG_MAX;
        for (int w = 0; w < kC; ++w)
          if (am_better(amv[w * 4 + ct], ami[w * 4 + ct], bv, bi)) {
            bv = amv[w * 4 + ct];
            bi = ami[w * 4 + ct];
          }
        p.am_val[bid * 4 + ct] = bv;
        p.am_idx[bid * 4 + ct] = bi;
      }
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
      s_flag = (atom_add_release(&p.sync[ph], 1u) == (unsigned)G - 1);
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

  // ---- the last CTA to finish the last phase wraps up the step
  if (s_flag) {
    __threadfence();
    if (ct < p.B) {
      if (p.run_head) {
        float bv = -INFINITY;
        long long bi = LLONG_MAX;
        for (int b = 0; b < G; ++b) {
          const float v = __ldcg(p.am_val + b * 4 + ct);
          const long long i = __ldcg(reinterpret_cast<const long long*>(p.am_idx) + b * 4 + ct);
          if (am_better(v, i, bv, bi)) {
            bv = v;
            bi = i;
          }
        }
        p.next[ct] = bi;
      }
      p.lens[ct] += 1;
    }
  }
}

// ======================================================================
bool pdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd) {
  if (hd != kHD || nkv <= 0 || nh % nkv != 0 || nh / nkv > kAGMax || nh > kNHMax) return false;
  if (H % 8 || I % 8 || qd % 8 || qkvd % 2 || V <= 0) return false;
  // every weight stage must fit a ring slot
  if ((size_t)I * 2 > kSlot || (size_t)H * 2 * 2 > kSlot) return false;
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
  Q2_CUDA_TRY(cudaFuncSetAttribute(pdecode_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)g.total));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
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
