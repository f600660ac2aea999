// linear.cu -- Y = X W^T (+ b) on CUDA cores: a warp-per-output-row GEMV
// for few rows of X (decode), and a 64x64-tiled GEMM for everything else.
// The weight layout is [out_features, in_features] as in the checkpoints.
// fp32 accumulation, one rounding of (sum + bias) to the output type.
// (LLAISYS final report, section 3.2: "linear"; bias optional.)
#include "common.cuh"
#include "gemm_tc.h"
#include "kernels.h"

namespace q2 {

// ------------------------------------------------------------------- GEMV
// One warp per output feature n; MT rows of X per pass (X is re-read from
// L1/L2, the weight row once per pass).
template <typename Tin, typename Tout, int MT>
__global__ void __launch_bounds__(256) gemv_kernel(Tout* __restrict__ y, const Tin* __restrict__ x,
                                                   const Tin* __restrict__ w,
                                                   const Tin* __restrict__ b, int M, int N, int K) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int V = Storage<Tin>::kVec;
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= N) return;
  const Tin* wr = w + (size_t)warp * K;
  float bias = b ? to_f(b[warp]) : 0.f;
  for (int m0 = 0; m0 < M; m0 += MT) {
    float acc[MT];
#pragma unroll
    for (int i = 0; i < MT; ++i) acc[i] = 0.f;
    for (int k = lane * V; k < K; k += 32 * V) {
      float wf[V];
      unpack16<Tin>(ld_stream16(wr + k), wf);
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        if (m0 + i < M) {
          float xf[V];
          unpack16<Tin>(__ldg(reinterpret_cast<const uint4*>(x + (size_t)(m0 + i) * K + k)), xf);
#pragma unroll
          for (int j = 0; j < V; ++j) acc[i] = fmaf(wf[j], xf[j], acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      float s = warp_sum(acc[i]);
      if (lane == 0 && m0 + i < M) y[(size_t)(m0 + i) * N + warp] = from_f<Tout>(s + bias);
    }
  }
}

// ------------------------------------------------------------- tiled GEMM
// 64x64 output tile per block of 256 threads, 4x4 outputs per thread, K in
// steps of 16 staged through shared memory (bounds-checked on every side).
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) gemm_simt_kernel(Tout* __restrict__ y,
                                                        const Tin* __restrict__ x,
                                                        const Tin* __restrict__ w,
                                                        const Tin* __restrict__ b, int M, int N,
                                                        int K) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float xs[BK][BM + 4];
  __shared__ float ws[BK][BN + 4];
  int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      int r = i / BK, c = i % BK;
      int gm = m0 + r, gk = k0 + c;
      xs[c][r] = (gm < M && gk < K) ? to_f(x[(size_t)gm * K + gk]) : 0.f;
      int gn = n0 + r;
      ws[c][r] = (gn < N && gk < K) ? to_f(w[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[kk][ty * 4 + i];
        bb[i] = ws[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn < N) y[(size_t)gm * N + gn] = from_f<Tout>(acc[i][j] + (b ? to_f(b[gn]) : 0.f));
    }
  }
}

template <typename Tin, typename Tout>
static q2_status linear_t(Tout* y, const Tin* x, const Tin* w, const Tin* b, int M, int N, int K,
                          cudaStream_t st, bool pdl) {
  constexpr int V = Storage<Tin>::kVec;
  bool vec_ok = (K % V == 0) && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w)) & 15) == 0;
  if (M <= 8 && vec_ok) {
    dim3 grid(ceil_div((long long)N * 32, 256));
    if (M == 1)
      Q2_LAUNCH(gemv_kernel<Tin, Tout, 1>, grid, dim3(256), 0, st, pdl, y, x, w, b, M, N, K);
    else if (M <= 2)
      Q2_LAUNCH(gemv_kernel<Tin, Tout, 2>, grid, dim3(256), 0, st, pdl, y, x, w, b, M, N, K);
    else if (M <= 4)
      Q2_LAUNCH(gemv_kernel<Tin, Tout, 4>, grid, dim3(256), 0, st, pdl, y, x, w, b, M, N, K);
    else
      Q2_LAUNCH(gemv_kernel<Tin, Tout, 8>, grid, dim3(256), 0, st, pdl, y, x, w, b, M, N, K);
    return Q2_OK;
  }
  dim3 grid(ceil_div(N, 64), ceil_div(M, 64));
  Q2_LAUNCH(gemm_simt_kernel<Tin, Tout>, grid, dim3(256), 0, st, pdl, y, x, w, b, M, N, K);
  return Q2_OK;
}

q2_status launch_linear(void* out, const void* in, const void* w, const void* b, int M, int N,
                        int K, int dtype, int out_dtype, cudaStream_t st, bool pdl) {
  if (M == 0 || N == 0) return Q2_OK;
  if (dtype == Q2_BF16) {
    using B = __nv_bfloat16;
    if (tc_linear_supported(M, N, K, out, in, w))
      return tc_linear(out, in, w, b, M, N, K, out_dtype, st, pdl);
    if (out_dtype == Q2_F32)
      return linear_t<B, float>((float*)out, (const B*)in, (const B*)w, (const B*)b, M, N, K, st, pdl);
    return linear_t<B, B>((B*)out, (const B*)in, (const B*)w, (const B*)b, M, N, K, st, pdl);
  }
  if (out_dtype != Q2_F32) {
    set_error("linear: fp32 inputs need an fp32 output");
    return Q2_ERR_DTYPE;
  }
  return linear_t<float, float>((float*)out, (const float*)in, (const float*)w, (const float*)b,
                                M, N, K, st, pdl);
}

}  // namespace q2
