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
// MOE_OK on an sm_100 device, else MOE_ERR_UNSUPPORTED with a message.
moe_status check_sm100();

// The calling thread's last-error text, and its reset at the start of every
// entry point.
const char* last_error_text();
void clear_last_error();

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Error bits written to the device error word.
enum : int {
  ERR_GEMM_TIMEOUT = 1,       // tcgen05 GEMM: an mbarrier wait ran out
  ERR_GEMM_FP8_TIMEOUT = 2,   // FP8 tcgen05 GEMM: an mbarrier wait ran out
  ERR_EP_BOUNDS = 4,          // expert-parallel copy: a row position past its buffer (skipped)
  ERR_GATHER_TIMEOUT = 8,     // row-gather pipeline (combine and its backward): a wait ran out
  ERR_BAD_OFFSETS = 16,       // group offsets outside [0, rows] or decreasing (clamped)
  ERR_BOUNDS = 32,            // checked build: an index outside its buffer (access skipped)
};

// ---------------------------------------------------------------- device side

// Checked build (-DMOE_CHECK_BOUNDS): internal indices are tested against the
// buffer they address before the access; a failed test records ERR_BOUNDS in
// the device error word and the access is skipped (no trap).  The release
// build compiles the tests away.
#ifdef MOE_CHECK_BOUNDS
__device__ __forceinline__ bool in_bounds(bool ok, int* err) {
  if (!ok) atomicOr(err, ERR_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ bool in_bounds(bool, int*) { return true; }
#endif

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

// The router's float32 affinity Sigmoid(x) = 1 / (1 + e^-x), with the fast
// exponential and division (a few 1e-7 from the exact value, well inside the
// tie-break's key-error bound).  Every kernel that forms a float32 key (the
// fused router, the top-K kernel, the tie-break's keys of unlisted experts)
// uses this one expression, so equal logits give equal keys everywhere.
__device__ __forceinline__ float router_affinity(float x) {
  return __fdividef(1.0f, 1.0f + __expf(-x));
}

// Row range [r0, r1) of group g from the caller's offsets, clamped so that
// 0 <= r0 <= r1 <= rows (offsets == nullptr: one group of all rows); a clamp
// that changes a value sets ERR_BAD_OFFSETS in *err (err may be null).
__device__ __forceinline__ void clamp_group_rows(const int32_t* offsets, int g, int rows, int* err,
                                                 int& r0, int& r1) {
  if (!offsets) {
    r0 = 0;
    r1 = rows;
    return;
  }
  const int a = __ldg(offsets + g), b = __ldg(offsets + g + 1);
  r0 = min(max(a, 0), rows);
  r1 = min(max(b, r0), rows);
  if (err && (r0 != a || r1 != b)) atomicOr(err, ERR_BAD_OFFSETS);
}

// roff[0..G] = the caller's group offsets made safe, by one whole warp: each
// value clamped to [0, rows] and raised to the largest earlier one, so the
// groups are disjoint row ranges inside [0, rows).  A change sets
// ERR_BAD_OFFSETS in *err.  offsets == nullptr: one group [0, rows).
__device__ __forceinline__ void load_offsets_warp(const int32_t* offsets, int G, int rows,
                                                  int* roff, int* err) {
  const int lane = threadIdx.x & 31;
  if (!offsets) {
    if (lane == 0) {
      roff[0] = 0;
      roff[1] = rows;
    }
    __syncwarp();
    return;
  }
  const int n = G + 1, per = (n + 31) / 32, j0 = lane * per;
  int run = 0;
  for (int i = 0; i < per; ++i) {
    const int j = j0 + i;
    if (j < n) {
      run = max(run, min(max(offsets[j], 0), rows));
      roff[j] = run;
    }
  }
  int incl = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl = max(incl, v);
  }
  int before = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) before = 0;
  bool bad = false;
  for (int i = 0; i < per; ++i) {
    const int j = j0 + i;
    if (j < n) {
      const int v = max(roff[j], before);
      bad |= v != offsets[j];
      roff[j] = v;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && err) atomicOr(err, ERR_BAD_OFFSETS);
  __syncwarp();
}

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
