// Router of the DeepSeekMoE layer ("DeepSeek-V3 技術報告", section 方法 / 2):
// affinity s_{i,t} = Sigmoid(u_t^T e_i), selection of the K largest s + b
// (g'-equation), gates normalised from the unbiased s of the selected
// experts, and the per-expert load that the bias rule reads.
//
// The logits come from a GEMM (tensor cores for bf16, CUDA cores for f32);
// this file holds the CUDA-core logits path and the per-token selection.
#include <math.h>

#include "launch.h"
#include "router_warp.cuh"

namespace moe {

moe_status launch_logits_simt(const void* u, const void* E, moe_dtype dt, int T, int d,
                              int N_r, float* logits, cudaStream_t s) {
  return launch_simt_gemm(u, E, 0, nullptr, 1, T, N_r, d, false, dt, logits, MOE_F32, s);
}

// Precise tie-break.  The tensor-core logits are float32 sums of d products,
// which can move s by a few 1e-6 at V3 width.  A token whose routing was
// decided by a key gap below the refine gap is listed together with the
// experts whose float32 key lies within the near distance of its close
// decisions; those experts get float64 logits (s = Sigmoid in float64,
// rounded once to float32: the affinity line's exact value) and the token is
// routed again.  The other experts keep their float32 keys, which are too far
// from every close decision for the float32 error to matter.  If the float64
// keys move the group choice, the experts of the new kept groups near the new
// (K+1)-th key get float64 keys as well.

// One warp per token (router_warp.cuh), the logits read from memory.
template <int V>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, int T,
                                                   int N_r, int K, int n_groups, int topk_groups,
                                                   int32_t* __restrict__ idx,
                                                   float* __restrict__ gate,
                                                   int32_t* __restrict__ counts, RefineLists rl,
                                                   float refine_gap, float near) {
  extern __shared__ int hist[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps_per_block = blockDim.x >> 5;
  (void)lane;
  float* wkeys = reinterpret_cast<float*>(hist + N_r) + warp * N_r;   // per-warp key staging
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int t = blockIdx.x * warps_per_block + warp; t < T; t += gridDim.x * warps_per_block)
    route_token_warp<V>(logits + (size_t)t * N_r, bias, t, N_r, K, n_groups, topk_groups, wkeys,
                        idx, gate, hist, rl, refine_gap, near, nullptr);
  __syncthreads();
  for (int i = threadIdx.x; i < N_r; i += blockDim.x)
    if (hist[i]) atomicAdd(&counts[i], hist[i]);
}

__device__ __forceinline__ float affinity64(double logit) {
  return (float)(1.0 / (1.0 + exp(-logit)));
}

// Float64 dot product of a token row and a centroid row by one warp: lane l
// takes the 16-byte vectors l, l + 32, ... of both rows, four at a time; the
// lanes' sums meet in a butterfly.  A product of two bfloat16 values is exact
// in float32 (8-bit significands) unless it falls below 2^-126, so each term
// needs one float64 conversion.
template <typename Tin>
__device__ __forceinline__ double warp_dot64(const Tin* __restrict__ x, const Tin* __restrict__ w,
                                             int nv, int lane) {
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  double a0 = 0.0, a1 = 0.0;
  for (int v0 = lane; v0 < nv; v0 += 32 * 4) {
    uint4 xv[4], wv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int v = v0 + 32 * q;
      xv[q] = v < nv ? x4[v] : make_uint4(0, 0, 0, 0);
      wv[q] = v < nv ? w4[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t xs[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
      const uint32_t ws[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
      if (sizeof(Tin) == 2) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          a0 += (double)(__uint_as_float(xs[k] << 16) * __uint_as_float(ws[k] << 16));
          a1 += (double)(__uint_as_float(xs[k] & 0xffff0000u) *
                         __uint_as_float(ws[k] & 0xffff0000u));
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          a0 = fma((double)__uint_as_float(xs[k]), (double)__uint_as_float(ws[k]), a0);
      }
    }
  }
  double a = a0 + a1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
  return a;
}

// Kept-group mask of keys held lane-strided (expert j*32 + lane in key[j]):
// a group's score is its largest key, the topk_groups best groups stay (ties
// to the lower group index).  wk: this warp's N_r floats of shared memory.
template <int V>
__device__ __forceinline__ unsigned warp_keep_groups(const float (&key)[V], float* wk, int N_r,
                                                     int n_groups, int topk_groups, int gs,
                                                     int lane) {
#pragma unroll
  for (int j = 0; j < V; ++j)
    if (j * 32 + lane < N_r) wk[j * 32 + lane] = key[j];
  __syncwarp();
  float gscore = -INFINITY;                       // lane g holds group g's score
  if (lane < n_groups)
    for (int i = 0; i < gs; ++i) gscore = fmaxf(gscore, wk[lane * gs + i]);
  __syncwarp();
  unsigned kept = 0;
  for (int r = 0; r < topk_groups; ++r) {
    float bk = (lane < n_groups && !((kept >> lane) & 1u)) ? gscore : -INFINITY;
    int bg = (lane < n_groups && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
      const int og = __shfl_xor_sync(0xffffffffu, bg, off);
      if (ok > bk || (ok == bk && og < bg)) { bk = ok; bg = og; }
    }
    kept |= 1u << bg;
  }
  return kept;
}

// Order-preserving keys of the eligible experts (0 = not eligible).
template <int V>
__device__ __forceinline__ void eligible_keys(const float (&key)[V], unsigned kept, int gs,
                                              int N_r, int lane, uint32_t (&ko)[V]) {
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int e = j * 32 + lane;
    ko[j] = (e < N_r && ((kept >> (e / gs)) & 1u)) ? ord_key(key[j]) : 0u;
  }
}

// The m-th largest eligible key (-inf if fewer than m are eligible).
template <int V>
__device__ __forceinline__ float warp_mth_key(uint32_t (&ko)[V], int m, int lane) {
  float out = -INFINITY;
  for (int k = 0; k < m; ++k) {
    uint32_t lb = 0u;
    int lj = 0;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (ko[j] > lb) { lb = ko[j]; lj = j; }
    const uint32_t mx = __reduce_max_sync(0xffffffffu, lb);
    if (mx == 0u) return -INFINITY;
    const int be = __reduce_min_sync(0xffffffffu, lb == mx ? lj * 32 + lane : 0x7fffffff);
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (j * 32 + lane == be) ko[j] = 0u;
    out = ord_float(mx);
  }
  return out;
}

// Expert e's float64 affinity into the lane that holds it.
template <int V>
__device__ __forceinline__ void set_key64(float (&sv)[V], float (&key)[V], uint32_t& r64, int e,
                                          float s64, const float* __restrict__ bias, int lane) {
  if ((e & 31) == lane) {
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (j == (e >> 5)) {
        sv[j] = s64;
        key[j] = s64 + bias[e];
        r64 |= 1u << j;
      }
  }
}

// Block slice of a float64 dot product: thread tid of the block adds the
// 16-byte vectors tid, tid + kRefineThreads, ... of both rows (eight loads in
// flight per operand); returns the thread's part.
constexpr int kRefineThreads = 128;          // four warps per listed token
constexpr int kRefineChunk = 8;              // listed experts per round of partial sums
template <typename Tin>
__device__ __forceinline__ double block_dot64_part(const Tin* __restrict__ x,
                                                   const Tin* __restrict__ w, int nv, int tid) {
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  double a0 = 0.0, a1 = 0.0;
  for (int v0 = tid; v0 < nv; v0 += kRefineThreads * 8) {
    uint4 xv[8], wv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int v = v0 + kRefineThreads * q;
      xv[q] = v < nv ? x4[v] : make_uint4(0, 0, 0, 0);
      wv[q] = v < nv ? w4[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t xs[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
      const uint32_t ws[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
      if (sizeof(Tin) == 2) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          a0 += (double)(__uint_as_float(xs[k] << 16) * __uint_as_float(ws[k] << 16));
          a1 += (double)(__uint_as_float(xs[k] & 0xffff0000u) *
                         __uint_as_float(ws[k] & 0xffff0000u));
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          a0 = fma((double)__uint_as_float(xs[k]), (double)__uint_as_float(ws[k]), a0);
      }
    }
  }
  return a0 + a1;
}

// One block of four warps per listed token.  Warp 0 holds the float32 keys of
// every expert (from the float32 logits, as the selection computed them);
// the four warps compute the float64 logits of the listed experts, each a
// quarter of every dot product, added in warp order; warp 0 takes the
// float64 keys, re-checks the group choice, redoes the selection, gates and
// load (a slot whose expert changed moves one unit of load) while the other
// warps start on the block's next token.
template <int V, typename Tin>
__global__ void __launch_bounds__(kRefineThreads) refine_token_kernel(
    const Tin* __restrict__ u, const Tin* __restrict__ E, const float* __restrict__ logits,
    const float* __restrict__ bias, int d, int N_r, int K, int n_groups, int topk_groups,
    RefineLists rl, float near, int32_t* __restrict__ idx, float* __restrict__ gate,
    int32_t* __restrict__ counts) {
  extern __shared__ float wk[];                         // [N_r] group-score staging (warp 0)
  __shared__ double part[kRefineThreads / 32][kRefineChunk];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  const int gs = grouped ? N_r / n_groups : N_r;
  const int nv = d / (16 / (int)sizeof(Tin));          // 16-byte vectors per row
  const int n = rl.hdr[0];
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int t = rl.tok[i], p0 = rl.start[i], np = rl.num[i];
    const Tin* ut = u + (size_t)t * d;
    float sv[V], key[V];
    uint32_t r64 = 0;                                  // bit j: key[j] is a float64 key
    unsigned kept32 = 1u;
    if (warp == 0) {
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = j * 32 + lane;
        if (e < N_r) {
          sv[j] = router_affinity(logits[(size_t)t * N_r + e]);
          key[j] = sv[j] + bias[e];
        } else {
          sv[j] = 0.f;
          key[j] = -INFINITY;
        }
      }
      if (grouped) kept32 = warp_keep_groups<V>(key, wk, N_r, n_groups, topk_groups, gs, lane);
    }
    for (int c0 = 0; c0 < np; c0 += kRefineChunk) {
      const int nc = min(kRefineChunk, np - c0);
      for (int c = 0; c < nc; ++c) {
        const int e = rl.pair[p0 + c0 + c] - t * N_r;
        double a = block_dot64_part<Tin>(ut, E + (size_t)e * d, nv, tid);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (lane == 0) part[warp][c] = a;
      }
      __syncthreads();
      if (warp == 0) {
        for (int c = 0; c < nc; ++c) {
          double a = 0.0;
#pragma unroll
          for (int w = 0; w < kRefineThreads / 32; ++w) a += part[w][c];
          set_key64<V>(sv, key, r64, rl.pair[p0 + c0 + c] - t * N_r, affinity64(a), bias, lane);
        }
      }
      __syncthreads();                                 // part is rewritten next
    }
    if (warp != 0) continue;
    unsigned kept = 1u;
    if (grouped) {
      kept = warp_keep_groups<V>(key, wk, N_r, n_groups, topk_groups, gs, lane);
      if (kept != kept32) {
        // the group choice moved: the new kept groups' experts near the new
        // (K+1)-th key join the float64 set (rare: warp 0 alone)
        uint32_t ko[V];
        eligible_keys<V>(key, kept, gs, N_r, lane, ko);
        const float thr = warp_mth_key<V>(ko, K + 1, lane) - near;
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const int e = j * 32 + lane;
          const bool add = e < N_r && ((kept >> (e / gs)) & 1u) && !((r64 >> j) & 1u) &&
                           key[j] >= thr;
          unsigned m = __ballot_sync(0xffffffffu, add);
          while (m) {
            const int ee = j * 32 + __ffs(m) - 1;
            m &= m - 1;
            const float s64 = affinity64(warp_dot64<Tin>(ut, E + (size_t)ee * d, nv, lane));
            set_key64<V>(sv, key, r64, ee, s64, bias, lane);
          }
        }
      }
    }
    // selection in the documented output order; lane k keeps the k-th winner
    uint32_t ko[V];
    eligible_keys<V>(key, grouped ? kept : 1u, gs, N_r, lane, ko);
    uint32_t lb = 0u;
    int lj = 0;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (ko[j] > lb) { lb = ko[j]; lj = j; }
    float sum = 0.f;
    int my_e = 0;
    float my_s = 0.f;
    for (int k = 0; k < K; ++k) {
      const uint32_t mx = __reduce_max_sync(0xffffffffu, lb);
      const int be = __reduce_min_sync(0xffffffffu, lb == mx ? lj * 32 + lane : 0x7fffffff);
      float s_win = 0.f;
      uint32_t nb = 0u;
      int nj = 0;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        if (j * 32 + lane == be) { s_win = sv[j]; ko[j] = 0u; }
        if (ko[j] > nb) { nb = ko[j]; nj = j; }
      }
      lb = nb;
      lj = nj;
      s_win = __shfl_sync(0xffffffffu, s_win, be & 31);
      sum += s_win;
      if (k < 32) {
        if (lane == k) { my_e = be; my_s = s_win; }
      } else if (lane == 0) {
        const size_t p = (size_t)t * K + k;
        const int was = idx[p];
        if (was != be) {
          atomicSub(&counts[was], 1);
          atomicAdd(&counts[be], 1);
          idx[p] = be;
        }
        gate[p] = s_win;
      }
    }
    if (lane < K) {
      const size_t p = (size_t)t * K + lane;
      const int was = idx[p];
      if (was != my_e) {
        atomicSub(&counts[was], 1);
        atomicAdd(&counts[my_e], 1);
        idx[p] = my_e;
      }
      gate[p] = my_s / sum;
    }
    if (K > 32) {
      __syncwarp();
      for (int k = 32 + lane; k < K; k += 32) {
        const size_t p = (size_t)t * K + k;
        gate[p] = gate[p] / sum;
      }
    }
  }
}

moe_status launch_refine(const void* u, const void* E, moe_dtype dt, const float* logits,
                         const float* b, int d, int N_r, int K, int n_groups, int topk_groups,
                         RefineLists rl, float near, int T, int32_t* idx, float* gate,
                         int32_t* counts, cudaStream_t s) {
  int blocks = T > 0 ? T : 1;                 // at most one block per token
  const int cap = 16 * sm_count();
  if (blocks > cap) blocks = cap;
  const size_t smem = (size_t)N_r * sizeof(float);   // warp 0's group-score staging
  const int V = (N_r + 31) / 32;
  const bool f32 = dt == MOE_F32;
#define MOE_REFINE_CASE(v)                                                                     \
  if (f32)                                                                                     \
    refine_token_kernel<v, float><<<blocks, kRefineThreads, smem, s>>>(                        \
        static_cast<const float*>(u), static_cast<const float*>(E), logits, b, d, N_r, K,      \
        n_groups, topk_groups, rl, near, idx, gate, counts);                                   \
  else                                                                                         \
    refine_token_kernel<v, __nv_bfloat16><<<blocks, kRefineThreads, smem, s>>>(                \
        static_cast<const __nv_bfloat16*>(u), static_cast<const __nv_bfloat16*>(E), logits, b, \
        d, N_r, K, n_groups, topk_groups, rl, near, idx, gate, counts);                        \
  break;
  switch (V <= 1 ? 1 : V <= 2 ? 2 : V <= 4 ? 4 : V <= 8 ? 8 : V <= 16 ? 16 : 32) {
    case 1: MOE_REFINE_CASE(1)
    case 2: MOE_REFINE_CASE(2)
    case 4: MOE_REFINE_CASE(4)
    case 8: MOE_REFINE_CASE(8)
    case 16: MOE_REFINE_CASE(16)
    default: MOE_REFINE_CASE(32)
  }
#undef MOE_REFINE_CASE
  return cuda_check(cudaGetLastError(), "refine_token_kernel launch");
}

moe_status launch_topk(const float* logits, const float* b, int T, int N_r, int K, int n_groups,
                       int topk_groups, int32_t* idx, float* gate, int32_t* counts,
                       RefineLists rl, float refine_gap, float near, cudaStream_t s) {
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
                                               gate, counts, rl, refine_gap, near);           \
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
