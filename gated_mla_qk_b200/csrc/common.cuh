// Shared device/host helpers for libgmla: element types, the device error
// flag, launch bookkeeping.  Nothing here is specific to one kernel.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/gmla.h"

namespace gmla {

// ---------------------------------------------------------------------------
// Element access: kernels are templated on the storage type T (float or
// __nv_bfloat16) and always compute in fp32.
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float ld(const T* p);
template <> __device__ __forceinline__ float ld<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ T cvt(float v);
template <> __device__ __forceinline__ float cvt<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Atomic max on a float in global memory whose initial value is a float
// (e.g. -inf).  Non-negative floats order like signed ints; negative floats
// order inversely like unsigned ints, so a signed max covers the first case
// and an unsigned min the second.  The result does not depend on the order in
// which blocks arrive.
__device__ __forceinline__ void atomic_max_float(float* addr, float v) {
  v += 0.f;  // -0 -> +0, so a zero maximum is not lost to the sign bit
  if (v >= 0.f) {
    atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
  } else {
    atomicMin(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
  }
}

// Device error flag: set by a bounded wait that gave up (value = status code).
// The library is one translation unit (gmla.cu includes every kernel header),
// so this single definition is the flag of every kernel.
__device__ int g_device_error = 0;

__device__ __forceinline__ void raise_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

// Wall-time limit of the device-side waits (mbarrier try_wait loops).  Waits
// inside one CTA normally last microseconds; one that lasts this long means
// the pipeline is broken, and the kernel gives up instead of hanging.  The
// limit of the pipeline waits is a device variable (gmla_set_wait_limit_ns
// shortens it, so that a test can make a wait run out); the drain waits a
// giving-up CTA runs for its own copies and MMAs keep the fixed limit.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ uint64_t g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ bool device_error_pending() {
  return *reinterpret_cast<volatile int*>(&g_device_error) != 0;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
void note_launches(int n);             // add to the process-wide launch counter
int cuda_status(cudaError_t e);        // GMLA_OK or GMLA_ECUDA (and remember e)
inline int check_launch() { return cuda_status(cudaGetLastError()); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dsize(gmla_dtype t) { return t == GMLA_BF16 ? 2 : 4; }

}  // namespace gmla
