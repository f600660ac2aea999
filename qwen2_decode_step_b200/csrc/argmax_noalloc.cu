// argmax_noalloc.cu -- q2_argmax_noalloc: the two-pass argmax of q2_argmax,
// with its pass-1 partials kept in a fixed array of the library's own device
// memory instead of memory requested from the CUDA allocator on each call.
//
// Why it exists: some callers cannot let a library allocate device memory at
// the moment they call it -- a host that has handed all device memory to its
// own pool and passes this library only its input and output buffers, a
// latency-critical loop that must not wait on the allocator, or code that
// records into a CUDA graph under a capture mode that refuses allocation
// calls.  q2_argmax takes its partials from cudaMallocAsync/cudaFreeAsync on
// every call; this entry point calls no allocator at all.
#include <map>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

// Room for 16384 (value, index) partials: 16384 * (8 + 4) bytes = 192 KiB,
// held by every GPU that loads the library until the process exits.
static constexpr size_t kMaxPartials = 16384;
static __device__ __align__(256) unsigned char
    g_argmax_scratch[kMaxPartials * (sizeof(int64_t) + sizeof(float))];

namespace {

std::mutex g_mu;
std::map<int, void*> g_scratch_addr;  // device -> device address of g_argmax_scratch

// The array's device address on the current device.  In host code the name
// g_argmax_scratch is only a host-side stand-in, so the address is asked of
// the runtime once per device (with that device current) and cached.
q2_status scratch_address(void** out) {
  int dev = 0;
  Q2_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_scratch_addr.find(dev);
  if (it != g_scratch_addr.end()) {
    *out = it->second;
    return Q2_OK;
  }
  void* p = nullptr;
  Q2_CUDA_TRY(cudaGetSymbolAddress(&p, g_argmax_scratch));
  g_scratch_addr[dev] = p;
  *out = p;
  return Q2_OK;
}

}  // namespace

using namespace q2;

extern "C" q2_status q2_argmax_noalloc(int64_t* max_idx, void* max_val, const void* vals,
                                       size_t rows, size_t n, int dtype, void* stream) {
  clear_error();
  Q2_CHECK_ARG(dtype == Q2_F32 || dtype == Q2_BF16, Q2_ERR_DTYPE, "dtype must be Q2_F32 or Q2_BF16");
  if (rows == 0) return Q2_OK;
  Q2_CHECK_ARG(max_idx && vals, Q2_ERR_INVALID_ARG, "argmax_noalloc: NULL pointer");
  Q2_CHECK_ARG(n > 0, Q2_ERR_SHAPE, "argmax_noalloc: empty rows");
  Q2_CHECK_ARG(rows <= kMaxPartials, Q2_ERR_CAPACITY,
               "argmax_noalloc: more than 16384 rows (the fixed partials array holds 16384 entries)");
  const int parts = argmax_parts(rows, n);
  Q2_CHECK_ARG(rows * (size_t)parts <= kMaxPartials, Q2_ERR_CAPACITY,
               "argmax_noalloc: rows x partials exceeds the fixed array of 16384 entries");
  void* base = nullptr;
  Q2_TRY(scratch_address(&base));
  // Pass 1 writes every one of the rows x parts partials before pass 2 reads
  // them, so nothing left over from an earlier call is ever read.
  int64_t* part_idx = static_cast<int64_t*>(base);
  float* part_val = reinterpret_cast<float*>(part_idx + kMaxPartials);
  return launch_argmax(max_idx, max_val, vals, rows, n, dtype, part_val, part_idx, parts,
                       as_stream(stream), false);
}
