// gemm_tc.cu -- bf16 GEMM on the sm_100a tensor cores.
#include "common.cuh"
#include "gemm_tc.h"

namespace q2 {

bool tc_linear_supported(int, int, int, const void*, const void*, const void*) { return false; }

q2_status tc_linear(void*, const void*, const void*, const void*, int, int, int, int, cudaStream_t,
                    bool) {
  set_error("tcgen05 linear not available");
  return Q2_ERR_STATE;
}

}  // namespace q2
