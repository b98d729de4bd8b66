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

// Precise tie-break.  The tensor-core logits are float32 sums of d products,
// which can move s by a few 1e-6 at V3 width.  A token whose routing was
// decided by a key gap below the refine gap is listed together with the
// experts whose float32 key lies within kRouterNearBoundary of one of its decision
// boundaries; those experts get float64 logits (s = Sigmoid in float64,
// rounded once to float32: the affinity line's exact value) and the token is
// routed again.  The other experts keep their float32 keys, which are too far
// below every boundary for the float32 error to matter.  If the group choice
// changes, every expert of the token is recomputed.

// Order-preserving map of a float key to an unsigned integer (every real key
// maps above 0; -0 is taken as +0, so equal keys map to equal integers).
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t b = __float_as_uint(f + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_float(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// One warp per token.  Lane l holds experts e = j*32 + l (j < V), so a
// token's logits are read with coalesced loads.  K rounds of a warp-wide
// arg-max with the order (key descending, index ascending) give the
// selection in the documented output order; lane k keeps the k-th winner
// (k < 32) so that the gates are normalised and written from registers.
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
                                                   int32_t* __restrict__ counts, RefineLists rl,
                                                   float refine_gap) {
  extern __shared__ int hist[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps_per_block = blockDim.x >> 5;
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  float* wkeys = reinterpret_cast<float*>(hist + N_r) + warp * N_r;   // per-warp key staging
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  for (int t = blockIdx.x * warps_per_block + warp; t < T; t += gridDim.x * warps_per_block) {
    float key[V], sv[V], kb[V];
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
      kb[j] = key[j];
    }
    float margin = INFINITY;     // smallest key gap that decided this token's routing
    float next_group = INFINITY; // score of the best group left out (group limit only)
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
      float last_kept = INFINITY;
      for (int r = 0; r <= topk_groups; ++r) {    // one extra round: the best excluded group
        float bk = (lane < n_groups && !((kept >> lane) & 1u)) ? gscore : -INFINITY;
        int bg = lane < n_groups && !((kept >> lane) & 1u) ? lane : 0x7fffffff;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
          const int og = __shfl_xor_sync(0xffffffffu, bg, off);
          if (ok > bk || (ok == bk && og < bg)) { bk = ok; bg = og; }
        }
        if (r < topk_groups) {
          kept |= 1u << bg;
          last_kept = bk;
        } else {
          margin = fminf(margin, last_kept - bk);   // kept vs excluded group scores
          next_group = bk;
        }
      }
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = j * 32 + lane;
        if (e < N_r && !((kept >> (e / gs)) & 1u)) key[j] = -INFINITY;
      }
    }
    // K+1 rounds of a warp arg-max on order-preserving integer keys: each
    // lane keeps the best of its own keys (ties to the lower index), the warp
    // takes the largest with one reduction and the lowest expert id holding it
    // with another; the winner's lane then drops it and rescans its keys.
    uint32_t ko[V];
#pragma unroll
    for (int j = 0; j < V; ++j) ko[j] = j * 32 + lane < N_r ? ord_key(key[j]) : 0u;
    uint32_t lb = 0u;
    int lj = 0;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (ko[j] > lb) { lb = ko[j]; lj = j; }
    float sum = 0.f, prev = INFINITY, next_key = -INFINITY;
    int my_e = 0;
    float my_s = 0.f;
    for (int k = 0; k <= K; ++k) {             // round K only measures the next key
      const uint32_t m = __reduce_max_sync(0xffffffffu, lb);
      if (m == 0u) break;                       // no key left (only after the K-th round)
      const int be = __reduce_min_sync(0xffffffffu, lb == m ? lj * 32 + lane : 0x7fffffff);
      const float bk = ord_float(m);
      margin = fminf(margin, prev - bk);        // adjacent selected keys, and K-th vs next
      prev = bk;
      if (k == K) { next_key = bk; break; }
      // the owner drops the winner (compared by expert id so that the arrays
      // stay in registers) and rescans; its unbiased s is broadcast
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
        idx[(size_t)t * K + k] = be;
        gate[(size_t)t * K + k] = s_win;
        atomicAdd(&hist[be], 1);
      }
    }
    if (lane < K) {
      idx[(size_t)t * K + lane] = my_e;
      gate[(size_t)t * K + lane] = my_s / sum;
      atomicAdd(&hist[my_e], 1);
    }
    if (K > 32) {
      __syncwarp();
      for (int k = 32 + lane; k < K; k += 32) {
        const size_t p = (size_t)t * K + k;
        gate[p] = gate[p] / sum;
      }
    }
    if (margin < refine_gap) {
      // list the token with every expert whose float32 key is near the lowest
      // key a decision hinged on (the (K+1)-th key inside the kept groups and,
      // with the group limit, the best excluded group's score)
      const float thr = fminf(next_key, next_group) - kRouterNearBoundary;
      int c = 0;
#pragma unroll
      for (int j = 0; j < V; ++j)
        if (j * 32 + lane < N_r && kb[j] >= thr) ++c;
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      int base = 0, slot = 0;
      if (lane == 0) {
        base = atomicAdd(&rl.hdr[1], total);
        slot = atomicAdd(&rl.hdr[0], 1);
        rl.tok[slot] = t;
        rl.start[slot] = base;
        rl.num[slot] = total;
      }
      int w = __shfl_sync(0xffffffffu, base, 0) + incl - c;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = j * 32 + lane;
        if (e < N_r && kb[j] >= thr) rl.pair[w++] = t * N_r + e;
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N_r; i += blockDim.x)
    if (hist[i]) atomicAdd(&counts[i], hist[i]);
}

// Float64 dot product of one token row and one centroid row: each lane
// accumulates its share in two float64 accumulators; returns the lane's part.
template <typename Tin>
__device__ __forceinline__ double dot64_part(const Tin* __restrict__ ut,
                                             const Tin* __restrict__ er, int nv, int v0,
                                             int stride) {
  double a0 = 0.0, a1 = 0.0;
  const uint4* u4 = reinterpret_cast<const uint4*>(ut);
  const uint4* e4 = reinterpret_cast<const uint4*>(er);
  for (int vb = v0; vb < nv; vb += 8 * stride) {
    uint4 x[8], w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {         // eight independent 16-byte loads per operand in flight
      const int v = vb + q * stride;
      x[q] = v < nv ? u4[v] : make_uint4(0, 0, 0, 0);
      w[q] = v < nv ? e4[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t xs[4] = {x[q].x, x[q].y, x[q].z, x[q].w};
      const uint32_t ws[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
      if (sizeof(Tin) == 2) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a0 = fma((double)__uint_as_float(xs[i] << 16), (double)__uint_as_float(ws[i] << 16), a0);
          a1 = fma((double)__uint_as_float(xs[i] & 0xffff0000u),
                   (double)__uint_as_float(ws[i] & 0xffff0000u), a1);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          a0 = fma((double)__uint_as_float(xs[i]), (double)__uint_as_float(ws[i]), a0);
      }
    }
  }
  return a0 + a1;
}

__device__ __forceinline__ float affinity64(double logit) {
  return (float)(1.0 / (1.0 + exp(-logit)));
}

// s of one expert from a float64 logit, the whole warp on one dot product.
template <typename Tin>
__device__ __forceinline__ float exact_affinity_warp(const Tin* __restrict__ ut,
                                                     const Tin* __restrict__ er, int d, int lane) {
  double acc = dot64_part(ut, er, d / (16 / (int)sizeof(Tin)), lane, 32);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  return affinity64(acc);
}

// Warp-wide arg-max of (key desc, index asc) over keys held lane-strided in kv[].
__device__ __forceinline__ void warp_best(const float* kv, int N_r, int lane, float& bk, int& be) {
  bk = -INFINITY;
  be = 0x7fffffff;
  for (int e = lane; e < N_r; e += 32)
    if (kv[e] > bk || (kv[e] == bk && e < be)) { bk = kv[e]; be = e; }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
    if (ok > bk || (ok == bk && oe < be)) { bk = ok; be = oe; }
  }
}

// Group limit on keys kv[]: returns the kept-group mask (topk_groups best
// group maxima, ties to the lower group index).
__device__ __forceinline__ unsigned keep_groups(const float* kv, int N_r, int n_groups,
                                                int topk_groups, int lane) {
  const int gs = N_r / n_groups;
  float gscore = -INFINITY;
  if (lane < n_groups)
    for (int j = 0; j < gs; ++j) gscore = fmaxf(gscore, kv[lane * gs + j]);
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

// One block per listed token: the float64 affinities of its listed experts
// (one warp per expert), float32 keys for every other expert (from the
// float32 logits, as the selection computed them), then selection, gates and
// load redone; a changed group choice recomputes every expert in float64.
// A token's listed experts are pair[start, start + num) (t*N_r + e codes).
constexpr int kRefineThreads = 256;
template <typename Tin>
__global__ void __launch_bounds__(kRefineThreads) refine_token_kernel(
    const Tin* __restrict__ u, const Tin* __restrict__ E, const float* __restrict__ logits,
    const float* __restrict__ bias, int d, int N_r, int K, int n_groups, int topk_groups,
    RefineLists rl, int32_t* __restrict__ idx, float* __restrict__ gate,
    int32_t* __restrict__ counts) {
  extern __shared__ float sm_r[];
  float* sv = sm_r;            // s [N_r]
  float* kv = sv + N_r;        // key [N_r]
  float* kw = kv + N_r;        // scratch keys [N_r]
  float* s64 = kw + N_r;       // float64 affinity of listed expert c, rounded once [N_r]
  __shared__ int s_full;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  const int gs = grouped ? N_r / n_groups : N_r;
  const int n = rl.hdr[0];
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int t = rl.tok[i], p0 = rl.start[i], np = rl.num[i];
    for (int c = warp; c < np; c += nw) {
      const int e = rl.pair[p0 + c] - t * N_r;
      const float sf = exact_affinity_warp(u + (size_t)t * d, E + (size_t)e * d, d, lane);
      if (lane == 0) s64[c] = sf;
    }
    for (int e = threadIdx.x; e < N_r; e += blockDim.x) {
      const float sf = 1.0f / (1.0f + expf(-logits[(size_t)t * N_r + e]));   // as the selection
      sv[e] = sf;
      kw[e] = sf + bias[e];
    }
    __syncthreads();
    unsigned kept32 = 0xffffffffu;
    if (grouped && warp == 0) kept32 = keep_groups(kw, N_r, n_groups, topk_groups, lane);
    for (int c = threadIdx.x; c < np; c += blockDim.x) sv[rl.pair[p0 + c] - t * N_r] = s64[c];
    __syncthreads();
    for (int e = threadIdx.x; e < N_r; e += blockDim.x) kv[e] = sv[e] + bias[e];
    __syncthreads();
    if (grouped) {
      if (warp == 0) {
        const unsigned kept = keep_groups(kv, N_r, n_groups, topk_groups, lane);
        if (lane == 0) s_full = kept != kept32;   // group choice moved: refine every expert
      }
      __syncthreads();
      if (s_full) {
        for (int e = warp; e < N_r; e += nw) {
          const float sf = exact_affinity_warp(u + (size_t)t * d, E + (size_t)e * d, d, lane);
          if (lane == 0) { sv[e] = sf; kv[e] = sf + bias[e]; }
        }
      }
      __syncthreads();
    }
    if (warp == 0) {
      for (int e = lane; e < N_r; e += 32) kw[e] = kv[e];
      __syncwarp();
      if (grouped) {
        const unsigned kept = keep_groups(kw, N_r, n_groups, topk_groups, lane);
        for (int e = lane; e < N_r; e += 32)
          if (!((kept >> (e / gs)) & 1u)) kw[e] = -INFINITY;
        __syncwarp();
      }
      float sum = 0.f;
      for (int k = 0; k < K; ++k) {
        float bk;
        int be;
        warp_best(kw, N_r, lane, bk, be);
        const float s_win = sv[be];
        sum += s_win;
        __syncwarp();
        if (lane == 0) {
          const size_t p = (size_t)t * K + k;
          atomicSub(&counts[idx[p]], 1);
          atomicAdd(&counts[be], 1);
          idx[p] = be;
          gate[p] = s_win;
          kw[be] = -INFINITY;
        }
        __syncwarp();
      }
      for (int k = lane; k < K; k += 32) {
        const size_t p = (size_t)t * K + k;
        gate[p] = gate[p] / sum;
      }
    }
    __syncthreads();
  }
}

moe_status launch_refine(const void* u, const void* E, moe_dtype dt, const float* logits,
                         const float* b, int d, int N_r, int K, int n_groups, int topk_groups,
                         RefineLists rl, int T, int32_t* idx, float* gate, int32_t* counts,
                         cudaStream_t s) {
  int blocks = 2 * sm_count();
  if (blocks > T) blocks = T > 0 ? T : 1;
  const size_t smem = (size_t)4 * N_r * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = dt == MOE_F32
        ? cudaFuncSetAttribute(refine_token_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
        : cudaFuncSetAttribute(refine_token_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_check(e, "refine_token_kernel smem attribute");
  }
  if (dt == MOE_F32)
    refine_token_kernel<float><<<blocks, kRefineThreads, smem, s>>>(
        static_cast<const float*>(u), static_cast<const float*>(E), logits, b, d, N_r, K,
        n_groups, topk_groups, rl, idx, gate, counts);
  else
    refine_token_kernel<__nv_bfloat16><<<blocks, kRefineThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(u), static_cast<const __nv_bfloat16*>(E), logits, b, d,
        N_r, K, n_groups, topk_groups, rl, idx, gate, counts);
  return cuda_check(cudaGetLastError(), "refine_token_kernel launch");
}

moe_status launch_topk(const float* logits, const float* b, int T, int N_r, int K, int n_groups,
                       int topk_groups, int32_t* idx, float* gate, int32_t* counts,
                       RefineLists rl, float refine_gap, cudaStream_t s) {
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
                                               gate, counts, rl, refine_gap);                 \
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
