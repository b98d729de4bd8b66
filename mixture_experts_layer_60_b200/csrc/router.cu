// Router of the DeepSeekMoE layer ("DeepSeek-V3 技術報告", section 方法 / 2):
// affinity s_{i,t} = Sigmoid(u_t^T e_i), selection of the K largest s + b
// (g'-equation), gates normalised from the unbiased s of the selected
// experts, and the per-expert load that the bias rule reads.
//
// The logits come from a GEMM (tensor cores for bf16, CUDA cores for f32);
// this file holds the CUDA-core logits path and the per-token selection.
#include <math.h>

#include "launch.h"

namespace moe {

moe_status launch_logits_simt(const void* u, const void* E, moe_dtype dt, int T, int d,
                              int N_r, float* logits, cudaStream_t s) {
  return launch_simt_gemm(u, E, 0, nullptr, 1, T, N_r, d, false, dt, logits, MOE_F32, s);
}

// One warp per token.  Lane l holds experts e = j*32 + l (j < V), so a
// token's logits are read with coalesced loads.  K rounds of a warp-wide
// arg-max with the order (key descending, index ascending) give the
// selection in the documented output order.
//
// Group limit (n_groups > 1, topk_groups < n_groups): experts form n_groups
// groups of N_r/n_groups consecutive indices; a group's score is its largest
// key s+b; only the topk_groups best groups (ties to the lower group index)
// stay eligible.  This is the per-token node limit of "DeepSeek V3 & R1
// 論文研究", section Cross-Node All-to-All; the score rule is this library's
// reading (the pages give only the limit).
template <int V>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, int T,
                                                   int N_r, int K, int n_groups, int topk_groups,
                                                   int32_t* __restrict__ idx,
                                                   float* __restrict__ gate,
                                                   int32_t* __restrict__ counts) {
  extern __shared__ int hist[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps_per_block = blockDim.x >> 5;
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  float* wkeys = reinterpret_cast<float*>(hist + N_r) + warp * N_r;   // per-warp key staging
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  for (int t = blockIdx.x * warps_per_block + warp; t < T; t += gridDim.x * warps_per_block) {
    float key[V], sv[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int e = j * 32 + lane;
      if (e < N_r) {
        const float x = logits[(size_t)t * N_r + e];
        const float s = 1.0f / (1.0f + expf(-x));
        sv[j] = s;
        key[j] = s + bias[e];
      } else {
        sv[j] = 0.f;
        key[j] = -INFINITY;
      }
    }
    if (grouped) {
      const int gs = N_r / n_groups;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = j * 32 + lane;
        if (e < N_r) wkeys[e] = key[j];
      }
      __syncwarp();
      float gscore = -INFINITY;                       // lane g holds group g's score
      if (lane < n_groups)
        for (int i = 0; i < gs; ++i) gscore = fmaxf(gscore, wkeys[lane * gs + i]);
      __syncwarp();
      unsigned kept = 0;
      for (int r = 0; r < topk_groups; ++r) {
        float bk = (lane < n_groups && !((kept >> lane) & 1u)) ? gscore : -INFINITY;
        int bg = lane < n_groups && !((kept >> lane) & 1u) ? lane : 0x7fffffff;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
          const int og = __shfl_xor_sync(0xffffffffu, bg, off);
          if (ok > bk || (ok == bk && og < bg)) { bk = ok; bg = og; }
        }
        kept |= 1u << bg;
      }
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = j * 32 + lane;
        if (e < N_r && !((kept >> (e / gs)) & 1u)) key[j] = -INFINITY;
      }
    }
    float sum = 0.f;
    for (int k = 0; k < K; ++k) {
      // lane-local best
      float bk = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = j * 32 + lane;
        if (key[j] > bk || (key[j] == bk && e < be)) {
          if (e < N_r) { bk = key[j]; be = e; }
        }
      }
      // warp arg-max
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ok > bk || (ok == bk && oe < be)) { bk = ok; be = oe; }
      }
      // the owner removes the winner and broadcasts its unbiased s
      float s_win = 0.f;
      if ((be & 31) == lane) {
#pragma unroll
        for (int j = 0; j < V; ++j)
          if (j == (be >> 5)) { s_win = sv[j]; key[j] = -INFINITY; }
      }
      s_win = __shfl_sync(0xffffffffu, s_win, be & 31);
      sum += s_win;
      if (lane == 0) {
        idx[(size_t)t * K + k] = be;
        gate[(size_t)t * K + k] = s_win;
        atomicAdd(&hist[be], 1);
      }
    }
    __syncwarp();
    for (int k = lane; k < K; k += 32) {
      const size_t p = (size_t)t * K + k;
      gate[p] = gate[p] / sum;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N_r; i += blockDim.x)
    if (hist[i]) atomicAdd(&counts[i], hist[i]);
}

moe_status launch_topk(const float* logits, const float* b, int T, int N_r, int K, int n_groups,
                       int topk_groups, int32_t* idx, float* gate, int32_t* counts,
                       cudaStream_t s) {
  const int threads = 256;
  const int wpb = threads / 32;
  int blocks = (T + wpb - 1) / wpb;
  const int cap = 4 * sm_count();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const size_t smem = (size_t)N_r * sizeof(int) * (1 + threads / 32);   // histogram + key staging
  const int V = (N_r + 31) / 32;
#define MOE_TOPK_CASE(v)                                                                    \
  topk_kernel<v><<<blocks, threads, smem, s>>>(logits, b, T, N_r, K, n_groups, topk_groups, idx, \
                                               gate, counts);                                  \
  break;
  switch (V <= 1 ? 1 : V <= 2 ? 2 : V <= 4 ? 4 : V <= 8 ? 8 : V <= 16 ? 16 : 32) {
    case 1: MOE_TOPK_CASE(1)
    case 2: MOE_TOPK_CASE(2)
    case 4: MOE_TOPK_CASE(4)
    case 8: MOE_TOPK_CASE(8)
    case 16: MOE_TOPK_CASE(16)
    default: MOE_TOPK_CASE(32)
  }
#undef MOE_TOPK_CASE
  return cuda_check(cudaGetLastError(), "topk_kernel launch");
}

}  // namespace moe
