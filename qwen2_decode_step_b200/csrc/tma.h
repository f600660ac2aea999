// tma.h -- TMA tensor maps (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library needs no link-time libcuda symbols) and
// the device-side tiled-load wrapper.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/q2.h"

namespace q2 {

// A 2-D bf16 tensor [rows, cols] (cols contiguous, row pitch `pitch_bytes`)
// tiled in boxes of box_rows x box_cols elements; swizzle_bytes 0 / 64 / 128.
q2_status make_tmap_2d_bf16(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                            uint64_t pitch_bytes, uint32_t box_rows, uint32_t box_cols,
                            int swizzle_bytes);

// Tiled 2-D TMA load of one box at (x = column, y = row) into shared memory,
// completing on `bar` (transaction bytes).  The column coordinate must be a
// multiple of 8 for bf16 (16-byte alignment of the innermost coordinate);
// rows beyond the tensor read as zeros.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
      "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
      : "memory");
}

}  // namespace q2
