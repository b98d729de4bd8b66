// Dispatch permutation: groups the T*K (token, slot) pairs by expert, tokens
// ascending inside each group, and copies the token rows into that order.
// This is the dispatch step that hands every token to the routed experts
// FFN_i of the h'-equation ("DeepSeek-V3 技術報告", section 方法 / 2).
//
// Four launches:
//   1. chunk_hist   per 256-token chunk, how many pairs go to each expert
//   2. chunk_scan   offsets (exclusive scan of the load) and, per chunk and
//                   expert, the first grouped row the chunk writes
//   3. chunk_rank   stable rank of each pair inside its chunk -> perm_src, inv_row
//   4. scatter_rows one warp per token: read the row once, store it K times
//                   with 16-byte vectors (and the FP8 tile scales, if any)
#include "launch.h"

namespace moe {

static constexpr int kChunk = 256;  // tokens per chunk = threads per block of steps 1 and 3

static inline int n_chunks(int T) { return (T + kChunk - 1) / kChunk; }

size_t permute_ws_bytes(int T, int N_r) {
  // chunk_hist and chunk_base, [n_chunks, N_r] int32 each
  return 2 * align_up((size_t)n_chunks(T) * N_r * sizeof(int32_t), 256);
}

__global__ void __launch_bounds__(kChunk) chunk_hist_kernel(const int32_t* __restrict__ idx, int T,
                                                            int N_r, int K,
                                                            int32_t* __restrict__ chunk_hist) {
  extern __shared__ int h[];
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int c = blockIdx.x;
  const int t = c * kChunk + threadIdx.x;
  if (t < T)
    for (int k = 0; k < K; ++k) {
      const int e = idx[(size_t)t * K + k];
      if ((unsigned)e < (unsigned)N_r) atomicAdd(&h[e], 1);
    }
  __syncthreads();
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) chunk_hist[(size_t)c * N_r + i] = h[i];
}

// One block of >= N_r threads (<= 1024).  Thread e owns expert e.
__global__ void __launch_bounds__(1024) chunk_scan_kernel(const int32_t* __restrict__ chunk_hist,
                                                          int nch, int N_r,
                                                          int32_t* __restrict__ chunk_base,
                                                          int32_t* __restrict__ offsets) {
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  const int lane = e & 31, warp = e >> 5;
  int total = 0;
  if (e < N_r)
    for (int c = 0; c < nch; ++c) total += chunk_hist[(size_t)c * N_r + e];
  // block-wide exclusive scan of `total`
  int incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += v;
    }
    if (lane < nw) warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e < N_r) {
    offsets[e] = excl;
    if (e == N_r - 1) offsets[N_r] = excl + total;
    int run = excl;
    for (int c = 0; c < nch; ++c) {
      chunk_base[(size_t)c * N_r + e] = run;
      run += chunk_hist[(size_t)c * N_r + e];
    }
  }
}

// Stable rank: pair (t, k) with expert e lands on
//   chunk_base[c][e] + #(tokens of earlier warps of the chunk routed to e)
//                    + #(earlier lanes of this warp routed to e).
// A token never holds the same expert twice, so ordering by token is total,
// and a warp's tokens routed to e form one 32-bit lane mask: the counts are
// population counts of those masks.
__global__ void __launch_bounds__(kChunk) chunk_rank_kernel(const int32_t* __restrict__ idx, int T,
                                                            int N_r, int K,
                                                            const int32_t* __restrict__ chunk_base,
                                                            int32_t* __restrict__ perm_src,
                                                            int32_t* __restrict__ inv_row) {
  extern __shared__ unsigned lanes_of[];    // [kChunk/32][N_r]: lanes of warp w routed to e
  const int c = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = c * kChunk + threadIdx.x;
  for (int i = threadIdx.x; i < (kChunk / 32) * N_r; i += blockDim.x) lanes_of[i] = 0;
  __syncthreads();
  const int32_t* it = idx + (size_t)t * K;
  if (t < T)
    for (int k = 0; k < K; ++k) {
      const int e = it[k];
      if ((unsigned)e < (unsigned)N_r) atomicOr(&lanes_of[warp * N_r + e], 1u << lane);
    }
  __syncthreads();
  if (t < T) {
    const unsigned below = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
      const int e = it[k];
      if ((unsigned)e >= (unsigned)N_r) {     // not an expert id: the pair is left out
        inv_row[(size_t)t * K + k] = -1;
        continue;
      }
      int r = chunk_base[(size_t)c * N_r + e];
      for (int w = 0; w < warp; ++w) r += __popc(lanes_of[w * N_r + e]);
      r += __popc(lanes_of[warp * N_r + e] & below);
      perm_src[r] = t;
      inv_row[(size_t)t * K + k] = r;
    }
  }
}

// One warp per token: each 16-byte vector of the row is loaded once and
// stored to the token's K grouped rows.
__global__ void __launch_bounds__(256) scatter_rows_kernel(const uint4* __restrict__ u,
                                                           const float* __restrict__ u_scale,
                                                           const int32_t* __restrict__ inv_row,
                                                           int T, int nvec, int nscale, int K,
                                                           uint4* __restrict__ x_perm,
                                                           float* __restrict__ x_scale,
                                                           int* err) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int rows[16];  // K <= 16 on this path; larger K takes the generic loop below
  const int Kc = K < 16 ? K : 16;
  const long long R = (long long)T * K;   // rows of x_perm
#pragma unroll
  for (int k = 0; k < 16; ++k)
    if (k < Kc) {
      rows[k] = inv_row[(size_t)t * K + k];
      if (rows[k] >= 0 && !in_bounds(rows[k] < R, err)) rows[k] = -1;
    }
  const uint4* src = u + (size_t)t * nvec;
  int c = lane;
  for (; c + 96 < nvec; c += 128) {
    const uint4 v0 = src[c], v1 = src[c + 32], v2 = src[c + 64], v3 = src[c + 96];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < Kc && rows[k] >= 0) {
        uint4* dst = x_perm + (size_t)rows[k] * nvec;
        dst[c] = v0; dst[c + 32] = v1; dst[c + 64] = v2; dst[c + 96] = v3;
      }
    }
  }
  for (; c < nvec; c += 32) {
    const uint4 v = src[c];
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (k < Kc && rows[k] >= 0) x_perm[(size_t)rows[k] * nvec + c] = v;
  }
  for (int k = 16; k < K; ++k) {
    const int r = inv_row[(size_t)t * K + k];
    if (r < 0 || !in_bounds(r < R, err)) continue;
    for (int cc = lane; cc < nvec; cc += 32) x_perm[(size_t)r * nvec + cc] = src[cc];
  }
  if (u_scale) {
    for (int k = 0; k < K; ++k) {
      const int r = inv_row[(size_t)t * K + k];
      if (r < 0 || !in_bounds(r < R, err)) continue;
      for (int j = lane; j < nscale; j += 32)
        x_scale[(size_t)r * nscale + j] = u_scale[(size_t)t * nscale + j];
    }
  }
}

moe_status launch_permute(const void* u, const float* u_scale, int elem_bytes, const int32_t* idx,
                          int T, int d, int N_r, int K, void* x_perm, float* x_scale,
                          int32_t* offsets, int32_t* perm_src, int32_t* inv_row, void* ws,
                          cudaStream_t s) {
  const int nch = n_chunks(T);
  int32_t* chunk_hist = static_cast<int32_t*>(ws);
  int32_t* chunk_base =
      chunk_hist + align_up((size_t)nch * N_r * sizeof(int32_t), 256) / sizeof(int32_t);
  chunk_hist_kernel<<<nch, kChunk, N_r * sizeof(int), s>>>(idx, T, N_r, K, chunk_hist);
  const int scan_threads = (N_r + 31) / 32 * 32;
  chunk_scan_kernel<<<1, scan_threads, 0, s>>>(chunk_hist, nch, N_r, chunk_base, offsets);
  const size_t rank_smem = (size_t)(kChunk / 32) * N_r * sizeof(unsigned);
  if (rank_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(chunk_rank_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)rank_smem);
    if (e != cudaSuccess) return cuda_check(e, "chunk_rank_kernel smem attribute");
  }
  chunk_rank_kernel<<<nch, kChunk, rank_smem, s>>>(idx, T, N_r, K, chunk_base, perm_src, inv_row);
  if (!x_perm) return cuda_check(cudaGetLastError(), "permute index launches");
  const int nvec = (int)((size_t)d * elem_bytes / 16);
  const int wpb = 8;
  scatter_rows_kernel<<<(T + wpb - 1) / wpb, wpb * 32, 0, s>>>(
      static_cast<const uint4*>(u), u_scale, inv_row, T, nvec, u_scale ? d / 128 : 0, K,
      static_cast<uint4*>(x_perm), x_scale, device_error_word());
  return cuda_check(cudaGetLastError(), "permute launches");
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Allocation-free variant of moe_permute.
//
// Some callers cannot hand this library a workspace: code that runs inside a
// host framework which owns every device allocation (a caching allocator or a
// fixed arena it does not expose), or a loop that must not allocate device
// memory once it has started.  For them, the permutation's scratch (the
// per-chunk expert histograms and first rows, 2 * ceil(T/256) * N_r int32)
// lives in a file-scope device array of kNoAllocScratchBytes that every GPU
// loading this library holds until the process exits.
//
// In host code the array's name is only a host-side handle, so its device
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) on the first call there; make that first call before any
// stream capture.  The per-device cache is atomic, so host threads may race
// on the first lookup (they store the same address).  A cudaDeviceReset
// unloads the library's device arrays; the cached address is then stale, so
// the library must not be used across a reset.  All calls share the array:
// two calls whose work overlaps on the GPU (different streams, or different
// host threads) race on it.  Every word a call reads is first written by the
// same call, so nothing has to be cleared between calls.
#include <atomic>

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = 1u << 20;   // 1 MiB: T up to 131072 at N_r = 256
constexpr int kNoAllocMaxDevices = 64;

__device__ __align__(256) unsigned char g_permute_scratch[kNoAllocScratchBytes];
std::atomic<void*> g_permute_scratch_addr[kNoAllocMaxDevices];

moe_status permute_scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "moe_permute_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(MOE_ERR_UNSUPPORTED, "moe_permute_noalloc: device %d out of range", dev);
  void* p = g_permute_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess || !p)
      return cuda_check(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                        "moe_permute_noalloc: cudaGetSymbolAddress of the static scratch");
    g_permute_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const void* u, const float* u_scale, moe_dtype dt,
                                          const int32_t* topk_idx, int T, int d, int N_r, int K,
                                          void* x_perm, float* x_scale, int32_t* offsets,
                                          int32_t* perm_src, int32_t* inv_row, void* stream) {
  using namespace moe;
  clear_last_error();
  int eb = 0;
  moe_status st = validate_permute_args("moe_permute_noalloc", u, u_scale, dt, topk_idx, T, d,
                                        N_r, K, x_perm, x_scale, offsets, perm_src, inv_row, &eb);
  if (st != MOE_OK) return st;
  const size_t need = T > 0 ? permute_ws_bytes(T, N_r) : 0;
  if (need > kNoAllocScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_permute_noalloc: T=%d, N_r=%d needs %zu bytes of scratch, more than the "
                "%zu-byte static array; use moe_permute with a workspace",
                T, N_r, need, kNoAllocScratchBytes);
  st = check_sm100();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0)
    return cuda_check(cudaMemsetAsync(offsets, 0, (size_t)(N_r + 1) * sizeof(int32_t), s),
                      "zero offsets");
  void* scratch = nullptr;
  st = permute_scratch_address(&scratch);
  if (st != MOE_OK) return st;
  return launch_permute(u, dt == MOE_E4M3 ? u_scale : nullptr, eb, topk_idx, T, d, N_r, K, x_perm,
                        dt == MOE_E4M3 ? x_scale : nullptr, offsets, perm_src, inv_row, scratch, s);
}
