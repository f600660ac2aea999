// gemm_tc.cu -- bf16 GEMM on the sm_100a tensor cores: TMA tiles in
// 128-byte-swizzled shared memory, tcgen05.mma with the accumulator in tensor
// memory, tcgen05.ld epilogue.
//
// out[m, n] = sum_k x[m, k] * w[n, k] (+ bias[n]): the Y = X W^T of a linear
// layer whose weight is stored [out_features, in_features] (both operands
// K-major).  The MMA runs with the weight rows as its M side (a tile of 128
// output features) and the tokens as its N side (a tile of BN tokens), so one
// thread of the epilogue owns one output feature and writes, token by token,
// 32 consecutive features per warp store.
//
// Warp roles (320 threads, one CTA per SM, persistent over the tiles):
//   warp 0      TMA producer: a 128 x 64 weight box and a BN x 64 token box
//               per k-block into a kStages ring (full/empty mbarriers)
//   warp 1      allocates tensor memory and issues the MMAs (one thread);
//               tcgen05.commit frees a ring stage and, after a tile's last
//               k-block, publishes the accumulator
//   warps 2-9   epilogue: two warps per 32-lane TMEM quarter, each taking
//               alternate 32-column chunks: tcgen05.ld, bias, the epilogue
//               operator, conversion, stores; then release the accumulator
// The accumulator is double-buffered in tensor memory (2 x BN fp32 columns),
// so the epilogue of one tile overlaps the MMAs of the next.  Every wait is
// bounded: a wait that runs out records an error flag and the kernel carries
// on to its end.
#include "common.cuh"
#include "gemm_tc.h"
#include "tma.h"

namespace q2 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kBM = 128;       // output features per tile (MMA M)
constexpr int kBK = 64;        // k per stage: one 128-byte swizzle atom of bf16
constexpr int kTcEpiWarps = 8;                     // two per TMEM lane quarter
constexpr int kTcThreads = (2 + kTcEpiWarps) * 32;  // + the producer and MMA warps
constexpr uint64_t kTcDeadlineNs = 2000ull * 1000 * 1000;  // 2 s

__device__ __forceinline__ uint64_t tc_gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = tc_gtimer();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (tc_gtimer() - t0 > kTcDeadlineNs) return false;
  }
}

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled tile whose
// 8-row groups are 1024 bytes apart (what a TMA box of 64 bf16 columns with
// 128-byte swizzle lays down): start address, leading offset 16 B (unused
// when swizzled), stride offset 1024 B, descriptor version 1, swizzle mode 2.
__device__ __forceinline__ uint64_t sw128_desc(const void* smem_tile) {
  const uint64_t addr = smem_u32(smem_tile);
  return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = bn, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int bn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct TcArgs {
  int M, N, K;       // tokens, output features, reduction
  const bf16* bias;  // [N] or null
  void* out;         // [M][ldo]
  int ldo;
  int out_f32;       // 1: fp32 output, 0: bf16 (one rounding)
  int epi;           // TC_EPI_*
  int* err;          // bit 1: a wait ran out
  int splits;        // K splits (1: the epilogue runs in this kernel)
  int kb_per;        // k-blocks per split
  float* ws;         // splits > 1: fp32 partial sums [splits][M][N]
};

template <int BN, int STAGES>
struct TcSmem {
  static constexpr size_t kA = (size_t)kBM * kBK * 2;  // weight box
  static constexpr size_t kB = (size_t)BN * kBK * 2;   // token box
  static constexpr size_t kStage = kA + kB;
  static constexpr size_t kBars = (2 * STAGES + 4) * 8 + 16;
  static constexpr size_t kTotal = STAGES * kStage + kBars + 1024;  // + alignment slack
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx,
                   const TcArgs a) {
  using SM = TcSmem<BN, STAGES>;
  extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
  uint8_t* smem = tc_smem_raw + ((1024u - (smem_u32(tc_smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SM::kStage);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (a.N + kBM - 1) / kBM, tiles_m = (a.M + BN - 1) / BN;
  const int ntiles = tiles_n * tiles_m;
  const int nitems = ntiles * a.splits;  // (tile, K split) work items
  const int kblocks = (a.K + kBK - 1) / kBK;
  // two accumulators of BN columns; the allocation is a power of two >= 32
  constexpr uint32_t kCols = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  static_assert(BN % 32 == 0 && 2 * BN <= 512, "the epilogue reads 32-column chunks of two BN-column accumulators");

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kTcEpiWarps);  // one arrival per epilogue warp
    }
    fence_mbar_init();
  }
  if (warp == 1) {  // tensor memory for the two accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_base_s)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_base_s);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The weights do not depend on the kernel before this one in the stream
    // (launched with programmatic dependent launch, this kernel may start while
    // that one finishes): the first item's first stages get their weight boxes
    // before the wait, their token boxes after it.
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int early = 0;  // stages of the first item whose weight box is in flight
      if (blockIdx.x < nitems) {
        const int t = blockIdx.x;
        const int tile = t % ntiles, kb0 = (t / ntiles) * a.kb_per;
        const int kb1 = min(kblocks, kb0 + a.kb_per);
        const int n0 = (tile % tiles_n) * kBM;
        for (; early < STAGES && kb0 + early < kb1; ++early) {
          mbar_arrive_expect_tx(&full[early], (uint32_t)SM::kStage);
          tma_load_2d(smem + early * SM::kStage, &tw, (kb0 + early) * kBK, n0, &full[early]);
        }
      }
      pdl_wait();
      for (int t = blockIdx.x; t < nitems; t += gridDim.x) {
        const int tile = t % ntiles, kb0 = (t / ntiles) * a.kb_per;
        const int kb1 = min(kblocks, kb0 + a.kb_per);
        const int n0 = (tile % tiles_n) * kBM, m0 = (tile / tiles_n) * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          uint8_t* st = smem + s * SM::kStage;
          if (early > 0) {  // the weight box is in flight: the token box
            tma_load_2d(st + SM::kA, &tx, kb * kBK, m0, &full[s]);
            --early;
          } else {
            if (!tc_wait(&empty[s], ph ^ 1u)) atomicOr(a.err, 2);
            mbar_arrive_expect_tx(&full[s], (uint32_t)SM::kStage);
            tma_load_2d(st, &tw, kb * kBK, n0, &full[s]);
            tma_load_2d(st + SM::kA, &tx, kb * kBK, m0, &full[s]);
          }
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // every load of this CTA is issued: the next kernel may start its
      // prologue (it waits for this grid before touching its outputs)
      pdl_launch_dependents();
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BN);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int t = blockIdx.x; t < nitems; t += gridDim.x, ++it) {
        const int acc = it & 1;
        const int kb0 = (t / ntiles) * a.kb_per, kb1 = min(kblocks, kb0 + a.kb_per);
        // the epilogue has drained this accumulator (fresh barriers pass at once)
        if (!tc_wait(&acc_empty[acc], (uint32_t)(((it >> 1) & 1) ^ 1))) atomicOr(a.err, 2);
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!tc_wait(&full[s], ph)) atomicOr(a.err, 2);
          tc_fence_after();
          const uint8_t* st = smem + s * SM::kStage;
          const uint64_t da = sw128_desc(st), db = sw128_desc(st + SM::kA);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // 16 bf16 = 32 bytes along the swizzle atom
            tc_mma(d, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc, kb != kb0 || k != 0);
          tc_commit(&empty[s]);  // the stage is free once these MMAs are done
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        tc_commit(&acc_full[acc]);  // the tile's accumulator is complete
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();  // the residual it reads and the output it writes belong to the stream's order
    const int q = warp & 3;                    // the TMEM lane quarter this warp may access
    const int half = (warp - 2) / 4;           // which alternate 32-column chunks it takes
    int it = 0;
    for (int t = blockIdx.x; t < nitems; t += gridDim.x, ++it) {
      const int acc = it & 1;
      const int tile = t % ntiles, split = t / ntiles;
      const int n0 = (tile % tiles_n) * kBM, m0 = (tile / tiles_n) * BN;
      if (lane == 0 && !tc_wait(&acc_full[acc], (uint32_t)((it >> 1) & 1))) atomicOr(a.err, 2);
      __syncwarp();
      tc_fence_after();
      const int n = n0 + 32 * q + lane;  // this thread's output feature
      const float bn = (a.bias != nullptr && n < a.N) ? __bfloat162float(a.bias[n]) : 0.f;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 32 * half; c < BN; c += 64) {
        float v[32];
        tmem_ld32(tbase + (uint32_t)c, v);
        if (a.splits > 1) {  // partial sums; the finishing kernel adds them in split order
          float* w = a.ws + (size_t)split * a.M * a.N;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + c + j;
            if (m < a.M && n < a.N) w[(size_t)m * a.N + n] = v[j];
          }
        } else if (a.epi == TC_EPI_SWIGLU) {
          // Rows 2i (gate) and 2i + 1 (up) sit in adjacent lanes.  For each
          // pair of tokens the even lane finishes the first and the odd lane
          // the second, after swapping the one value each is missing.
          const bool odd = (lane & 1) != 0;
          const bool pair_ok = (n | 1) < a.N;
          bf16* col = reinterpret_cast<bf16*>(a.out) + (n >> 1);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float mine0 = round_st<bf16>(v[j] + bn), mine1 = round_st<bf16>(v[j + 1] + bn);
            const float got = __shfl_xor_sync(0xffffffffu, odd ? mine0 : mine1, 1);
            const float gv = odd ? got : mine0, uv = odd ? mine1 : got;
            const int m = m0 + c + j + (odd ? 1 : 0);
            if (pair_ok && m < a.M)
              col[(size_t)m * a.ldo] = from_f<bf16>(uv * (gv / (1.0f + expf(-gv))));
          }
        } else if (a.epi == TC_EPI_RESID) {
          // all 32 residual loads first (they do not depend on the stores)
          bf16* col = reinterpret_cast<bf16*>(a.out) + (size_t)(m0 + c) * a.ldo + n;
          const bool nok = n < a.N;
          float xr[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            xr[j] = (nok && m0 + c + j < a.M) ? __bfloat162float(col[(size_t)j * a.ldo]) : 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (nok && m0 + c + j < a.M) col[(size_t)j * a.ldo] = from_f<bf16>(xr[j] + round_st<bf16>(v[j] + bn));
        } else if (a.out_f32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + c + j;
            if (m < a.M && n < a.N) reinterpret_cast<float*>(a.out)[(size_t)m * a.ldo + n] = v[j] + bn;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + c + j;
            if (m < a.M && n < a.N)
              reinterpret_cast<bf16*>(a.out)[(size_t)m * a.ldo + n] = from_f<bf16>(v[j] + bn);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols)
                 : "memory");
  }
}

// Split-K finish: y = sum of the splits' partials in split order (+ bias),
// then the epilogue.  One thread per output element (per gate/up pair for
// SwiGLU).
__global__ void tc_finish_kernel(const TcArgs a) {
  pdl_launch_dependents();
  pdl_wait();  // the partials are the GEMM's (launched just before it)
  const int N = a.N;
  const int cols = a.epi == TC_EPI_SWIGLU ? N / 2 : N;
  const size_t total = (size_t)a.M * cols;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(i / cols), c = (int)(i % cols);
    if (a.epi == TC_EPI_SWIGLU) {
      float g = 0.f, u = 0.f;
      for (int s = 0; s < a.splits; ++s) {
        const float* w = a.ws + ((size_t)s * a.M + m) * N;
        g += w[2 * c];
        u += w[2 * c + 1];
      }
      if (a.bias) {
        g += __bfloat162float(a.bias[2 * c]);
        u += __bfloat162float(a.bias[2 * c + 1]);
      }
      const float gv = round_st<bf16>(g), uv = round_st<bf16>(u);
      reinterpret_cast<bf16*>(a.out)[(size_t)m * a.ldo + c] = from_f<bf16>(uv * (gv / (1.0f + expf(-gv))));
    } else {
      float y = 0.f;
      for (int s = 0; s < a.splits; ++s) y += a.ws[((size_t)s * a.M + m) * N + c];
      if (a.bias) y += __bfloat162float(a.bias[c]);
      if (a.epi == TC_EPI_RESID) {
        bf16* o = reinterpret_cast<bf16*>(a.out) + (size_t)m * a.ldo + c;
        *o = from_f<bf16>(__bfloat162float(*o) + round_st<bf16>(y));
      } else if (a.out_f32) {
        reinterpret_cast<float*>(a.out)[(size_t)m * a.ldo + c] = y;
      } else {
        reinterpret_cast<bf16*>(a.out)[(size_t)m * a.ldo + c] = from_f<bf16>(y);
      }
    }
  }
}

template <int BN, int STAGES>
q2_status tc_launch(const CUtensorMap& tw, const CUtensorMap& tx, const TcArgs& a, cudaStream_t st) {
  using SM = TcSmem<BN, STAGES>;
  Q2_CUDA_TRY(cudaFuncSetAttribute(tc_gemm_kernel<BN, STAGES>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kTotal));
  const int items = ((a.N + kBM - 1) / kBM) * ((a.M + BN - 1) / BN) * a.splits;
  const int grid = items < num_sms() ? items : num_sms();
  // programmatic dependent launch: the kernel waits (griddepcontrol.wait)
  // before it touches anything the kernels before it produce
  const cudaError_t le = launch_k(tc_gemm_kernel<BN, STAGES>, dim3(grid), dim3(kTcThreads), SM::kTotal, st, true,
                                  tw, tx, a);
  if (le != cudaSuccess) {
    set_error(std::string("tcgen05 gemm launch: ") + cudaGetErrorString(le));
    return Q2_ERR_CUDA;
  }
  if (a.splits > 1) {
    const size_t total = (size_t)a.M * (a.epi == TC_EPI_SWIGLU ? a.N / 2 : a.N);
    const int blocks = (int)((total + 255) / 256 < (size_t)num_sms() * 8 ? (total + 255) / 256 : num_sms() * 8);
    const cudaError_t fe = launch_k(tc_finish_kernel, dim3(blocks), dim3(256), 0, st, true, a);
    if (fe != cudaSuccess) {
      set_error(std::string("tcgen05 gemm finish launch: ") + cudaGetErrorString(fe));
      return Q2_ERR_CUDA;
    }
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("tcgen05 gemm launch: ") + cudaGetErrorString(e));
    return Q2_ERR_CUDA;
  }
  return Q2_OK;
}

}  // namespace

bool tc_linear_supported(int M, int N, int K, const void* out, const void* in, const void* w) {
  if (M < 64 || N < kBM || K < kBK || K % 8 != 0) return false;  // TMA: 16-byte row pitch
  const uintptr_t al = reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(w);
  (void)out;
  return (al & 15) == 0;
}

// Token tile: 256 wide from 256 tokens up (narrower tiles fill the last wave
// better but raise the operand traffic per FLOP; 128 measured slower), 192
// when that cuts the wave-quantised work by a tenth or more: ceil(tiles /
// SMs) x BN, e.g. 1536 features x 4096 tokens, 192 tiles of 256 (two waves,
// the second a third full) against 264 of 192 (two waves).
int tc_gemm_token_tile(int M, int N, int sms) {
  if (M < 128) return 64;
  if (M < 256) return 128;
  const long long tn = (N + kBM - 1) / kBM;
  const long long w256 = (tn * ((M + 255) / 256) + sms - 1) / sms * 256;
  const long long w192 = (tn * ((M + 191) / 192) + sms - 1) / sms * 192;
  return 10 * w192 <= 9 * w256 ? 192 : 256;
}

q2_status tc_gemm(void* out, int ldo, int out_dtype, int epi, const void* x, const void* w,
                  const void* bias, int M, int N, int K, cudaStream_t st, int* err, float* ws,
                  size_t ws_bytes) {
  if (M <= 0 || N <= 0) return Q2_OK;
  if (K % 8 != 0 || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(w) & 15)) {
    set_error("tcgen05 gemm: K must be a multiple of 8 and operands 16-byte aligned");
    return Q2_ERR_INVALID_ARG;
  }
  if (epi == TC_EPI_SWIGLU && (N % 2 != 0 || out_dtype != Q2_BF16)) {
    set_error("tcgen05 gemm: the SwiGLU epilogue needs an even N and a bf16 output");
    return Q2_ERR_INVALID_ARG;
  }
  if (!err) {
    set_error("tcgen05 gemm: no error word");
    return Q2_ERR_INVALID_ARG;
  }
  TcArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.bias = reinterpret_cast<const bf16*>(bias);
  a.out = out;
  a.ldo = ldo;
  a.out_f32 = out_dtype == Q2_F32;
  a.epi = epi;
  a.err = err;
  const int bn = tc_gemm_token_tile(M, N, num_sms());
  // Split K when the tiles alone would leave SMs idle (few output features,
  // few tokens): aim for one work item per SM, at least two k-blocks each,
  // within the workspace.
  const int tiles = ((N + kBM - 1) / kBM) * ((M + bn - 1) / bn);
  const int kblocks = (K + kBK - 1) / kBK;
  int splits = 1;
  if (ws != nullptr && tiles < num_sms()) {
    splits = (num_sms() + tiles - 1) / tiles;
    if (splits > kblocks / 2) splits = kblocks / 2;
    while (splits > 1 && (size_t)splits * M * N * sizeof(float) > ws_bytes) --splits;
    if (splits < 1) splits = 1;
  }
  a.kb_per = (kblocks + splits - 1) / splits;
  a.splits = (kblocks + a.kb_per - 1) / a.kb_per;  // every split has a k-block
  a.ws = ws;
  CUtensorMap tw, tx;
  Q2_TRY(make_tmap_2d_bf16(&tw, w, (uint64_t)N, (uint64_t)K, (uint64_t)K * 2, kBM, kBK, 128));
  Q2_TRY(make_tmap_2d_bf16(&tx, x, (uint64_t)M, (uint64_t)K, (uint64_t)K * 2, (uint32_t)bn, kBK, 128));
  if (bn == 256) return tc_launch<256, 4>(tw, tx, a, st);
  if (bn == 192) return tc_launch<192, 5>(tw, tx, a, st);
  if (bn == 128) return tc_launch<128, 6>(tw, tx, a, st);
  return tc_launch<64, 8>(tw, tx, a, st);
}

q2_status tc_linear(void* out, const void* in, const void* w, const void* bias, int M, int N, int K,
                    int out_dtype, cudaStream_t st, bool pdl) {
  (void)pdl;
  return tc_gemm(out, N, out_dtype, TC_EPI_PLAIN, in, w, bias, M, N, K, st, op_error_flag(), nullptr, 0);
}

}  // namespace q2
