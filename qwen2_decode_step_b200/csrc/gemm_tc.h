// gemm_tc.h -- bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM, TMA).
#pragma once

#include <cuda_runtime.h>

#include "../../include/q2.h"

namespace q2 {

// Whether the tcgen05 path takes this linear (bf16 in, M large enough, K and
// N multiples of the tile, pointers aligned for TMA).
bool tc_linear_supported(int M, int N, int K, const void* out, const void* in, const void* w);
// out[M, N] (out_dtype) = in[M, K] . w[N, K]^T (+ bias[N]), bf16 operands.
q2_status tc_linear(void* out, const void* in, const void* w, const void* bias, int M, int N, int K,
                    int out_dtype, cudaStream_t st, bool pdl);

}  // namespace q2
