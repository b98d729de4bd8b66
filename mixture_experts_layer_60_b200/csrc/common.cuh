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

// Raises a kernel's dynamic shared-memory limit to `bytes` once per device
// (done: a per-call-site array of kMaxSmemDevices flags).
constexpr int kMaxSmemDevices = 64;
moe_status ensure_max_smem(const void* kernel, int bytes, bool* done, const char* what);

// Number of SMs of the current device (cached per device).
int sm_count();

// True when the current device is compute capability 10.0 (sm_100a kernels).
bool device_is_sm100();

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Error bits written to the device error word.
enum : int {
  ERR_GEMM_TIMEOUT = 1,       // tcgen05 GEMM: an mbarrier wait ran out
  ERR_GEMM_FP8_TIMEOUT = 2,   // FP8 tcgen05 GEMM: an mbarrier wait ran out
  ERR_EP_BOUNDS = 4,          // expert-parallel copy: a row position past its buffer (skipped)
  ERR_GATHER_TIMEOUT = 8,     // row-gather pipeline (combine and its backward): a wait ran out
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

// 8 bf16 or 4 f32 lanes per 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  static __device__ __forceinline__ uint4 store(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint4 store(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

}  // namespace moe
