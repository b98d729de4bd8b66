// Internal helpers shared by the CUDA translation units of libmoe.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- host side

// Records a formatted message as the calling thread's last error and returns `st`.
moe_status fail(moe_status st, const char* fmt, ...);

// Wraps a CUDA runtime result: MOE_OK, or MOE_ERR_CUDA with the runtime's text.
moe_status cuda_check(cudaError_t e, const char* what);

// Device address of the library's device error word on the current device
// (one int per device, set by kernels that give up a bounded wait).
int* device_error_word();

// Number of SMs of the current device (cached per device).
int sm_count();

// True when the current device is compute capability 10.0 (sm_100a kernels).
bool device_is_sm100();

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Error bits written to the device error word.
enum : int {
  ERR_GEMM_TIMEOUT = 1,       // tcgen05 GEMM: an mbarrier wait ran out
  ERR_GEMM_FP8_TIMEOUT = 2,   // FP8 tcgen05 GEMM: an mbarrier wait ran out
};

// ---------------------------------------------------------------- device side

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> struct IO;
template <> struct IO<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ float cvt(float v) { return v; }
  static __device__ __forceinline__ float to(float v) { return v; }
};
template <> struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float cvt(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 to(float v) { return __float2bfloat16_rn(v); }
};

}  // namespace moe
