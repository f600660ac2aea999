// common.cuh -- internal helpers shared by the library's CUDA sources:
// status plumbing, storage-type traits, and thin wrappers over the sm_90+/
// sm_100a PTX the kernels use (programmatic dependent launch, mbarriers,
// cp.async and bulk copies).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/q2.h"

namespace q2 {

// ------------------------------------------------------------------ status
void set_error(const std::string& msg);
void clear_error();

#define Q2_CHECK_ARG(cond, code, msg) \
  do {                                \
    if (!(cond)) {                    \
      ::q2::set_error(msg);           \
      return (code);                  \
    }                                 \
  } while (0)

#define Q2_CUDA_TRY(expr)                                                              \
  do {                                                                                 \
    cudaError_t _e = (expr);                                                           \
    if (_e != cudaSuccess) {                                                           \
      ::q2::set_error(std::string(#expr) + ": " + cudaGetErrorString(_e));             \
      return (_e == cudaErrorMemoryAllocation) ? Q2_ERR_OOM : Q2_ERR_CUDA;             \
    }                                                                                  \
  } while (0)

#define Q2_TRY(expr)                  \
  do {                                \
    q2_status _s = (expr);            \
    if (_s != Q2_OK) return _s;       \
  } while (0)

// Last launch error of the calling thread, as a status.
q2_status launch_status(const char* what);

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Library-wide device error word of the per-operator kernels.  One per device
// that loads the library.  Every error word (this one and each model's) uses
// the same bits: value 1 = a token id outside [0, vocab); value 2 = a
// bounded device-side wait ran out (a pipeline or grid-phase dependency that
// never arrived).
int* op_error_flag();
constexpr int kErrIndex = 1;
constexpr int kErrTimeout = 2;

// The status (and message) of a nonzero error word: Q2_ERR_TIMEOUT if a wait
// ran out (it takes precedence: the results are undefined), else
// Q2_ERR_INDEX.  `who` prefixes the message.
q2_status device_error_status(int bits, const char* who);

// ------------------------------------------------------------ storage types
template <typename T>
struct Storage;
template <>
struct Storage<float> {
  static constexpr int kDtype = Q2_F32;
  static constexpr int kVec = 4;  // elements per 16-byte vector
};
template <>
struct Storage<__nv_bfloat16> {
  static constexpr int kDtype = Q2_BF16;
  static constexpr int kVec = 8;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Round through the storage type (the write-back an operator boundary does).
template <typename T>
__device__ __forceinline__ float round_st(float x) {
  return to_f(from_f<T>(x));
}

// 16-byte vector <-> floats.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& v, float* f);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& v, float* f) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <typename T>
__device__ __forceinline__ uint4 pack16(const float* f);
template <>
__device__ __forceinline__ uint4 pack16<float>(const float* f) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}
template <>
__device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&p);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Streaming 16-byte load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---------------------------------------------- programmatic dependent launch
// griddepcontrol.wait blocks until the preceding grid in the stream has
// completed and its memory is visible; launch_dependents lets the next grid
// start launching.  Both are no-ops without the PDL launch attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and the caller must record an error and bail
// out) if the phase does not complete within `limit` polls.  Every spin in
// this library is bounded.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint32_t limit = 1u << 26) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Bulk copy global -> shared through the TMA engine, completing on `bar`.
// Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same with an L2 eviction hint for data streamed once (weights).
__device__ __forceinline__ void bulk_g2s_evict_first(void* smem_dst, const void* gmem_src,
                                                     uint32_t bytes, uint64_t* bar,
                                                     uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Ampere-style 16-byte async copy with zero fill (src_bytes = 0 -> zeros).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// (value, index) pair order for argmax: larger value first, then the lower
// index; a NaN ranks above every number and the first NaN wins.
__device__ __forceinline__ bool am_better(float v, long long i, float bv, long long bi) {
  bool vn = isnan(v), bn = isnan(bv);
  if (vn || bn) return (vn && bn) ? (i < bi) : vn;
  if (v > bv) return true;
  if (v < bv) return false;
  return i < bi;
}

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

int num_sms();

}  // namespace q2

namespace q2 {
// Launch with an optional programmatic-dependent-launch attribute.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
}  // namespace q2

#define Q2_LAUNCH(...)                                                            \
  do {                                                                            \
    cudaError_t _le = ::q2::launch_k(__VA_ARGS__);                                \
    if (_le != cudaSuccess) {                                                     \
      ::q2::set_error(std::string("kernel launch: ") + cudaGetErrorString(_le)); \
      return Q2_ERR_CUDA;                                                         \
    }                                                                             \
  } while (0)
