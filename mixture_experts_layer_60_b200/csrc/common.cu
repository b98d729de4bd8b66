// Host-side helpers: error text, CUDA result checks, per-device caches.
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace moe {

namespace {
thread_local char g_last_error[512] = "";
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int* g_err_word_addr[kMaxDevices] = {nullptr};
int g_is_sm100[kMaxDevices] = {0};  // 0 unknown, 1 yes, 2 no
}  // namespace

// One error word per device; kernels that give up a bounded wait set a bit.
__device__ int g_device_error_word = 0;

moe_status fail(moe_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

moe_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MOE_OK;
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int* device_error_word() {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  if (!g_err_word_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    g_err_word_addr[dev] = static_cast<int*>(p);
  }
  return g_err_word_addr[dev];
}

moe_status ensure_max_smem(const void* kernel, int bytes, bool* done, const char* what) {
  const int dev = current_device();
  if (dev < 0) return fail(MOE_ERR_CUDA, "%s: no current device", what);
  if (done[dev]) return MOE_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_check(e, what);
  done[dev] = true;
  return MOE_OK;
}

int sm_count() {
  const int dev = current_device();
  if (dev < 0) return 148;
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

bool device_is_sm100() {
  const int dev = current_device();
  if (dev < 0) return false;
  if (!g_is_sm100[dev]) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    g_is_sm100[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return g_is_sm100[dev] == 1;
}

moe_status check_sm100() {
  if (!device_is_sm100())
    return fail(MOE_ERR_UNSUPPORTED, "libmoe kernels need an sm_100 (B200) device");
  return MOE_OK;
}

const char* last_error_text() { return g_last_error; }
void clear_last_error() { g_last_error[0] = 0; }

}  // namespace moe
