// gemm_tc.h -- bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM, TMA).
#pragma once

#include <cuda_runtime.h>

#include "../../include/q2.h"

namespace q2 {

// Epilogues of tc_gemm (y = x w^T + bias, per output element):
//   TC_EPI_PLAIN   out[m][n] = y (bf16 with one rounding, or fp32)
//   TC_EPI_SWIGLU  w holds gate/up rows interleaved (row 2j gate j, row 2j + 1
//                  up j): out[m][j] = silu(bf16(y[2j])) * bf16(y[2j + 1]), bf16
//   TC_EPI_RESID   out[m][n] = bf16(out[m][n] + bf16(y)) (residual add in place)
enum { TC_EPI_PLAIN = 0, TC_EPI_SWIGLU = 1, TC_EPI_RESID = 2 };

// Whether the tcgen05 path takes this linear (bf16 operands, M >= 64 tokens,
// N >= 128 features, K a multiple of 8, operands 16-byte aligned).
bool tc_linear_supported(int M, int N, int K, const void* out, const void* in, const void* w);
// The token tile width (BN) tc_gemm takes for M tokens x N features on a
// machine of `sms` SMs: 64 or 128 below 256 tokens, else 256, or 192 where
// that cuts ceil(tiles / sms) x BN by a tenth.  Host only.
int tc_gemm_token_tile(int M, int N, int sms);
// out[M, N] (out_dtype) = in[M, K] . w[N, K]^T (+ bias[N]), bf16 operands.
// A pipeline wait that runs out sets value 2 in the operators' error word.
q2_status tc_linear(void* out, const void* in, const void* w, const void* bias, int M, int N, int K,
                    int out_dtype, cudaStream_t st, bool pdl);
// The general form: output row stride `ldo` (elements) and an epilogue.  With
// a workspace (fp32, `ws_bytes`), a product with fewer tiles than SMs splits
// K across CTAs; the partial sums are added in a fixed order by a second
// kernel, so results do not depend on scheduling.  A pipeline wait that runs
// out (a deadline on the global timer) sets value 2 in the device word `err`
// (the caller's error word: the model's, or the operators').
q2_status tc_gemm(void* out, int ldo, int out_dtype, int epi, const void* x, const void* w,
                  const void* bias, int M, int N, int K, cudaStream_t st, int* err,
                  float* ws = nullptr, size_t ws_bytes = 0);

}  // namespace q2
