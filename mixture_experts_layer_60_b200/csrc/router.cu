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
// experts whose float32 key lies within the near distance of one of its decision
// boundaries; those experts get float64 logits (s = Sigmoid in float64,
// rounded once to float32: the affinity line's exact value) and the token is
// routed again.  The other experts keep their float32 keys, which are too far
// below every boundary for the float32 error to matter.  If the group choice
// changes, every expert of the token is recomputed.

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

// One block per listed token: the float64 affinities of its listed experts,
// float32 keys for every other expert (from the float32 logits, as the
// selection computed them), then selection, gates and load redone.  A token's
// listed experts are pair[start, start + num) (t*N_r + e codes): every key
// down to `near` under the lowest key a decision hinged on.  When the float64
// keys move the group choice, the experts of the new kept groups whose key
// lies within `near` of the new (K+1)-th key get float64 affinities too; a
// float32 key further below is, within the key error bound, truly below it.
//
// The dot products are split by slices of d: warp w holds slice w of the
// token row in registers (kSliceVecs 16-byte vectors per lane at most) and
// adds up that slice of the listed experts' rows, kDotsPerPass experts per
// pass with all their loads in flight; the partial sums of an expert are
// added in warp order.  Every step of a token is a few dependent memory
// round trips: the block reads its pair list, token slice and logits row at
// once, then one round trip per pass, then the selection in shared memory.
constexpr int kRefineThreads = 512;
constexpr int kRefineWarps = kRefineThreads / 32;
constexpr int kSliceVecs = 4;      // d <= 16 * 32 * 4 * vector width (16384 bf16 elements)
constexpr int kDotsPerPass = 4;

// Slice `v0 .. v0 + nv_slice` (16-byte vectors) of the dot products of the
// token row (this lane's part in xv) with experts ex[c0 .. c0 + kDotsPerPass)
// (the last one repeated past n); lane 0 stores them to part_w[c].
template <typename Tin>
__device__ __forceinline__ void slice_dots(const uint4 (&xv)[kSliceVecs], const Tin* __restrict__ E,
                                           int d, const int* ex, int c0, int n, int v0,
                                           int nv_slice, int lane, double* part_w) {
  const uint4* er[kDotsPerPass];
#pragma unroll
  for (int q = 0; q < kDotsPerPass; ++q)
    er[q] = reinterpret_cast<const uint4*>(E + (size_t)ex[min(c0 + q, n - 1)] * d) + v0;
  uint4 w[kSliceVecs][kDotsPerPass];
#pragma unroll
  for (int i = 0; i < kSliceVecs; ++i) {
    const int v = lane + 32 * i;
#pragma unroll
    for (int q = 0; q < kDotsPerPass; ++q)
      w[i][q] = v < nv_slice ? er[q][v] : make_uint4(0, 0, 0, 0);
  }
  double acc[kDotsPerPass];
#pragma unroll
  for (int q = 0; q < kDotsPerPass; ++q) {
    double a = 0.0;
#pragma unroll
    for (int i = 0; i < kSliceVecs; ++i) {
      const uint32_t xs[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
      const uint32_t ws[4] = {w[i][q].x, w[i][q].y, w[i][q].z, w[i][q].w};
      if (sizeof(Tin) == 2) {
        // a product of two bfloat16 values is exact in float32 (8-bit
        // significands) unless it falls below 2^-126, so one float64
        // conversion per term suffices
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          a += (double)(__uint_as_float(xs[k] << 16) * __uint_as_float(ws[k] << 16));
          a += (double)(__uint_as_float(xs[k] & 0xffff0000u) *
                        __uint_as_float(ws[k] & 0xffff0000u));
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          a = fma((double)__uint_as_float(xs[k]), (double)__uint_as_float(ws[k]), a);
      }
    }
    acc[q] = a;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int q = 0; q < kDotsPerPass; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], off);
  if (lane == 0)
#pragma unroll
    for (int q = 0; q < kDotsPerPass; ++q)
      if (c0 + q < n) part_w[c0 + q] = acc[q];
}

template <typename Tin>
__global__ void __launch_bounds__(kRefineThreads, 1) refine_token_kernel(
    const Tin* __restrict__ u, const Tin* __restrict__ E, const float* __restrict__ logits,
    const float* __restrict__ bias, int d, int N_r, int K, int n_groups, int topk_groups,
    RefineLists rl, float near, int32_t* __restrict__ idx, float* __restrict__ gate,
    int32_t* __restrict__ counts) {
  extern __shared__ float sm_r[];
  float* sv = sm_r;            // s [N_r]
  float* kv = sv + N_r;        // key [N_r]
  float* kw = kv + N_r;        // scratch keys [N_r]
  double* part = reinterpret_cast<double*>(kw + N_r + (N_r & 1));   // [kRefineWarps][N_r]
  int* lst = reinterpret_cast<int*>(part + kRefineWarps * N_r);     // [N_r] listed experts
  int* is64 = lst + N_r;       // [N_r] float64 already
  int* more = is64 + N_r;      // [N_r] experts to add; the new selection at the end
  float* ngate = reinterpret_cast<float*>(part);                    // [K] at the end
  __shared__ int s_full, s_more;
  __shared__ unsigned s_kept;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool grouped = n_groups > 1 && topk_groups < n_groups;
  const int gs = grouped ? N_r / n_groups : N_r;
  const int nv = d / (16 / (int)sizeof(Tin));          // 16-byte vectors per row
  const int nv_slice = (nv + kRefineWarps - 1) / kRefineWarps;
  const int v0 = warp * nv_slice;
  const int my_nv = max(0, min(nv_slice, nv - v0));
  double* part_w = part + warp * N_r;
  const int n = rl.hdr[0];
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int t = rl.tok[i], p0 = rl.start[i], np = rl.num[i];
    // the pair list, this warp's slice of the token row and the float32 keys
    // (as the selection computed them), all loads issued together
    for (int c = threadIdx.x; c < np; c += blockDim.x) lst[c] = rl.pair[p0 + c] - t * N_r;
    uint4 xv[kSliceVecs];
    const uint4* ut4 = reinterpret_cast<const uint4*>(u + (size_t)t * d) + v0;
#pragma unroll
    for (int k = 0; k < kSliceVecs; ++k) {
      const int v = lane + 32 * k;
      xv[k] = v < my_nv ? ut4[v] : make_uint4(0, 0, 0, 0);
    }
    for (int e = threadIdx.x; e < N_r; e += blockDim.x) {
      const float sf = router_affinity(logits[(size_t)t * N_r + e]);
      sv[e] = sf;
      kw[e] = sf + bias[e];
    }
    __syncthreads();
    for (int c = 0; c < np; c += kDotsPerPass)
      slice_dots<Tin>(xv, E, d, lst, c, np, v0, my_nv, lane, part_w);
    unsigned kept32 = 0xffffffffu;
    if (grouped && warp == 0) kept32 = keep_groups(kw, N_r, n_groups, topk_groups, lane);
    __syncthreads();
    for (int c = threadIdx.x; c < np; c += blockDim.x) {
      double a = 0.0;
      for (int w = 0; w < kRefineWarps; ++w) a += part[w * N_r + c];
      sv[lst[c]] = affinity64(a);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N_r; e += blockDim.x) kv[e] = sv[e] + bias[e];
    __syncthreads();
    if (grouped) {
      if (warp == 0) {
        const unsigned kept = keep_groups(kv, N_r, n_groups, topk_groups, lane);
        if (lane == 0) {
          s_full = kept != kept32;
          s_kept = kept;
        }
      }
      for (int e = threadIdx.x; e < N_r; e += blockDim.x) is64[e] = 0;
      __syncthreads();
      if (s_full) {
        // the group choice moved: the new kept groups' experts near the new
        // (K+1)-th key join the float64 set
        for (int c = threadIdx.x; c < np; c += blockDim.x) is64[lst[c]] = 1;
        __syncthreads();
        if (warp == 0) {
          const unsigned kept = s_kept;
          for (int e = lane; e < N_r; e += 32)
            kw[e] = ((kept >> (e / gs)) & 1u) ? kv[e] : -INFINITY;
          __syncwarp();
          float bk = -INFINITY;
          int be;
          for (int k = 0; k <= K; ++k) {        // bk: the (K+1)-th key, -inf if none
            warp_best(kw, N_r, lane, bk, be);
            if (bk == -INFINITY) break;
            __syncwarp();
            if (lane == 0) kw[be] = -INFINITY;
            __syncwarp();
          }
          const float thr = bk - near;
          int m = 0;
          for (int e0 = 0; e0 < N_r; e0 += 32) {
            const int e = e0 + lane;
            const bool add = e < N_r && ((kept >> (e / gs)) & 1u) && !is64[e] && kv[e] >= thr;
            const unsigned bal = __ballot_sync(0xffffffffu, add);
            if (add) more[m + __popc(bal & ((1u << lane) - 1u))] = e;
            m += __popc(bal);
          }
          if (lane == 0) s_more = m;
        }
        __syncthreads();
        const int nm = s_more;
        for (int c = 0; c < nm; c += kDotsPerPass)
          slice_dots<Tin>(xv, E, d, more, c, nm, v0, my_nv, lane, part_w);
        __syncthreads();
        for (int c = threadIdx.x; c < nm; c += blockDim.x) {
          double a = 0.0;
          for (int w = 0; w < kRefineWarps; ++w) a += part[w * N_r + c];
          const int e = more[c];
          sv[e] = affinity64(a);
          kv[e] = sv[e] + bias[e];
        }
      }
      __syncthreads();
    }
    if (warp == 0) {
      // selection on the refined keys; the new experts and unnormalised gates
      // go to shared memory, then lanes k < K rewrite their slots and move
      // the load counts of the slots whose expert changed
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
          more[k] = be;
          ngate[k] = s_win;
          kw[be] = -INFINITY;
        }
        __syncwarp();
      }
      for (int k = lane; k < K; k += 32) {
        const size_t p = (size_t)t * K + k;
        const int was = idx[p], now = more[k];
        if (was != now) {
          atomicSub(&counts[was], 1);
          atomicAdd(&counts[now], 1);
          idx[p] = now;
        }
        gate[p] = ngate[k] / sum;
      }
    }
    __syncthreads();
  }
}

moe_status launch_refine(const void* u, const void* E, moe_dtype dt, const float* logits,
                         const float* b, int d, int N_r, int K, int n_groups, int topk_groups,
                         RefineLists rl, float near, int T, int32_t* idx, float* gate,
                         int32_t* counts, cudaStream_t s) {
  int blocks = sm_count();
  if (blocks > T) blocks = T > 0 ? T : 1;
  if ((size_t)d * (dt == MOE_F32 ? 4 : 2) > (size_t)kRefineWarps * 32 * kSliceVecs * 16)
    return fail(MOE_ERR_UNSUPPORTED, "router tie-break: d=%d is too long", d);
  const size_t smem = (size_t)(3 * N_r + (N_r & 1)) * sizeof(float) +
                      (size_t)kRefineWarps * N_r * sizeof(double) + 3 * (size_t)N_r * sizeof(int);
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
        n_groups, topk_groups, rl, near, idx, gate, counts);
  else
    refine_token_kernel<__nv_bfloat16><<<blocks, kRefineThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(u), static_cast<const __nv_bfloat16*>(E), logits, b, d,
        N_r, K, n_groups, topk_groups, rl, near, idx, gate, counts);
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
