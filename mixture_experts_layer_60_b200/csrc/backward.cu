// Per-token kernels of the layer backward: the gradient of the h'-equation
// through the combine, the gate normalisation and the affinity of
// "DeepSeek-V3 技術報告" (section 方法 / 2), and the unpermute that sums the
// input gradient.  The selection is held fixed (it is piecewise constant in
// s + b); gradients reach s only through g = s_sel / sum(s_sel).
//
//   dy_perm[r(t,k)] = g_{t,k} dh'_t                    (upstream of expert idx(t,k))
//   dg_{t,k}        = <dh'_t, y_perm[r(t,k)]>
//   ds_{t,k}        = (dg_{t,k} - sum_j g_{t,j} dg_{t,j}) / sum_j s_{t,j}
//   dlogit_{t,k}    = ds_{t,k} s_{t,k} (1 - s_{t,k}),   s = Sigmoid(u_t . e_idx)
//   du_t = dh'_t + sum_j dxs_j[t] + sum_k dx_perm[r(t,k)] + sum_k dlogit_{t,k} e_idx(t,k)
//   dE_i = sum over rows r of expert i of dlogit_perm[r] x(r)   (x_perm, or u gathered)
#include "launch.h"

namespace moe {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per token.  Reads dh'_t, u_t, the K rows y_perm[r] and the K rows
// e_idx once; writes the K rows dy_perm[r] and the per-slot scalars.
template <typename E, int KMAX>
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const uint4* __restrict__ dh, const uint4* __restrict__ u, const uint4* __restrict__ Ew,
    const uint4* __restrict__ yp, const int32_t* __restrict__ inv_row,
    const int32_t* __restrict__ idx, const float* __restrict__ gate, int T, int nvec, int K,
    uint4* __restrict__ dyp, float* __restrict__ d_gate, float* __restrict__ d_logit,
    float* __restrict__ d_logit_perm) {
  constexpr int N = Vec<E>::N;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int rows[KMAX], ex[KMAX];
  float g[KMAX], dg[KMAX], lg[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    dg[k] = 0.f;
    lg[k] = 0.f;
    if (k < K) {
      rows[k] = inv_row[(size_t)t * K + k];
      ex[k] = idx[(size_t)t * K + k];
      g[k] = gate[(size_t)t * K + k];
    }
  }
  for (int c = lane; c < nvec; c += 32) {
    float fd[N], fu[N], tmp[N];
    Vec<E>::load(dh[(size_t)t * nvec + c], fd);
    Vec<E>::load(u[(size_t)t * nvec + c], fu);
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K) {
        Vec<E>::load(yp[(size_t)rows[k] * nvec + c], tmp);
#pragma unroll
        for (int i = 0; i < N; ++i) dg[k] = fmaf(fd[i], tmp[i], dg[k]);
        Vec<E>::load(Ew[(size_t)ex[k] * nvec + c], tmp);
#pragma unroll
        for (int i = 0; i < N; ++i) lg[k] = fmaf(fu[i], tmp[i], lg[k]);
#pragma unroll
        for (int i = 0; i < N; ++i) tmp[i] = g[k] * fd[i];
        dyp[(size_t)rows[k] * nvec + c] = Vec<E>::store(tmp);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    if (k < K) {
      dg[k] = warp_sum(dg[k]);
      lg[k] = warp_sum(lg[k]);
    }
  }
  if (lane == 0) {
    float S = 0.f, gdg = 0.f, s[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K) {
        s[k] = 1.0f / (1.0f + expf(-lg[k]));
        S += s[k];
        gdg = fmaf(g[k], dg[k], gdg);
      }
    }
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K) {
        const float ds = (dg[k] - gdg) / S;
        const float dl = ds * s[k] * (1.0f - s[k]);
        d_gate[(size_t)t * K + k] = dg[k];
        d_logit[(size_t)t * K + k] = dl;
        d_logit_perm[rows[k]] = dl;
      }
    }
  }
}

// One warp per token: du_t = dh'_t + sum_j dxs_j[t] + sum_k dx_perm[r] + sum_k dlogit_k e_idx,
// summed in float32 in that order and rounded once.
template <typename E, int KMAX>
__global__ void __launch_bounds__(256) unpermute_backward_kernel(
    const uint4* __restrict__ dh, const uint4* __restrict__ dxs, int N_s,
    const uint4* __restrict__ dxp, const int32_t* __restrict__ inv_row,
    const int32_t* __restrict__ idx, const float* __restrict__ d_logit,
    const uint4* __restrict__ Ew, int T, int nvec, int K, uint4* __restrict__ du) {
  constexpr int N = Vec<E>::N;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int rows[KMAX], ex[KMAX];
  float dl[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    if (k < K) {
      rows[k] = inv_row[(size_t)t * K + k];
      ex[k] = idx[(size_t)t * K + k];
      dl[k] = d_logit[(size_t)t * K + k];
    }
  }
  for (int c = lane; c < nvec; c += 32) {
    float acc[N], tmp[N];
    Vec<E>::load(dh[(size_t)t * nvec + c], acc);
    for (int j = 0; j < N_s; ++j) {
      Vec<E>::load(dxs[((size_t)j * T + t) * nvec + c], tmp);
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] += tmp[i];
    }
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K) {
        Vec<E>::load(dxp[(size_t)rows[k] * nvec + c], tmp);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] += tmp[i];
      }
    }
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K) {
        Vec<E>::load(Ew[(size_t)ex[k] * nvec + c], tmp);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = fmaf(dl[k], tmp[i], acc[i]);
      }
    }
    du[(size_t)t * nvec + c] = Vec<E>::store(acc);
  }
}

// dE[i, cols] for one expert i and 128 16-byte column vectors per block:
// each thread owns one vector and walks the expert's rows in order.
template <typename E>
__global__ void __launch_bounds__(128) router_weight_grad_kernel(
    const uint4* __restrict__ xp, const int32_t* __restrict__ x_rows,
    const float* __restrict__ dlp, const int32_t* __restrict__ offsets, int nvec,
    float* __restrict__ dE) {
  constexpr int N = Vec<E>::N;
  const int e = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= nvec) return;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  float acc[N], tmp[N];
#pragma unroll
  for (int i = 0; i < N; ++i) acc[i] = 0.f;
  for (int r = r0; r < r1; ++r) {
    const float w = dlp[r];
    const size_t row = x_rows ? (size_t)x_rows[r] : (size_t)r;
    Vec<E>::load(xp[row * nvec + c], tmp);
#pragma unroll
    for (int i = 0; i < N; ++i) acc[i] = fmaf(w, tmp[i], acc[i]);
  }
  float4* out = reinterpret_cast<float4*>(dE + (size_t)e * nvec * N + (size_t)c * N);
#pragma unroll
  for (int i = 0; i < N / 4; ++i)
    out[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
}

}  // namespace

template <typename E>
static moe_status combine_bwd_dispatch(const void* dh, const void* u, const void* Ew,
                                       const void* yp, const int32_t* inv_row,
                                       const int32_t* idx, const float* gate, int T, int d, int K,
                                       void* dyp, float* d_gate, float* d_logit,
                                       float* d_logit_perm, cudaStream_t s) {
  const int nvec = d / Vec<E>::N;
  const int wpb = 8;
  dim3 grid((T + wpb - 1) / wpb), block(wpb * 32);
  auto c4 = [](const void* p) { return static_cast<const uint4*>(p); };
  if (K <= 8)
    combine_backward_kernel<E, 8><<<grid, block, 0, s>>>(
        c4(dh), c4(u), c4(Ew), c4(yp), inv_row, idx, gate, T, nvec, K, static_cast<uint4*>(dyp),
        d_gate, d_logit, d_logit_perm);
  else
    combine_backward_kernel<E, 16><<<grid, block, 0, s>>>(
        c4(dh), c4(u), c4(Ew), c4(yp), inv_row, idx, gate, T, nvec, K, static_cast<uint4*>(dyp),
        d_gate, d_logit, d_logit_perm);
  return cuda_check(cudaGetLastError(), "combine_backward launch");
}

moe_status launch_combine_backward(const void* dh, const void* u, const void* E,
                                   const void* y_perm, const int32_t* inv_row,
                                   const int32_t* idx, const float* gate, moe_dtype dt, int T,
                                   int d, int K, void* dy_perm, float* d_gate, float* d_logit,
                                   float* d_logit_perm, cudaStream_t s) {
  const long long rb = (long long)d * (dt == MOE_F32 ? 4 : 2);
  if (gather_pipe_supported(GATHER_COMBINE_BWD, 0, K, rb))
    return launch_gather_pipe(GATHER_COMBINE_BWD, dt, dh, u, nullptr, 0, y_perm,
                              (long long)T * K, E, inv_row, idx, gate, T, K, rb, dy_perm, d_gate,
                              d_logit, d_logit_perm, s);
  if (dt == MOE_F32)
    return combine_bwd_dispatch<float>(dh, u, E, y_perm, inv_row, idx, gate, T, d, K, dy_perm,
                                       d_gate, d_logit, d_logit_perm, s);
  return combine_bwd_dispatch<__nv_bfloat16>(dh, u, E, y_perm, inv_row, idx, gate, T, d, K,
                                             dy_perm, d_gate, d_logit, d_logit_perm, s);
}

template <typename E>
static moe_status unpermute_bwd_dispatch(const void* dh, const void* dxs, int N_s,
                                         const void* dxp, const int32_t* inv_row,
                                         const int32_t* idx, const float* d_logit, const void* Ew,
                                         int T, int d, int K, void* du, cudaStream_t s) {
  const int nvec = d / Vec<E>::N;
  const int wpb = 8;
  dim3 grid((T + wpb - 1) / wpb), block(wpb * 32);
  auto c4 = [](const void* p) { return static_cast<const uint4*>(p); };
  if (K <= 8)
    unpermute_backward_kernel<E, 8><<<grid, block, 0, s>>>(
        c4(dh), c4(dxs), N_s, c4(dxp), inv_row, idx, d_logit, c4(Ew), T, nvec, K,
        static_cast<uint4*>(du));
  else
    unpermute_backward_kernel<E, 16><<<grid, block, 0, s>>>(
        c4(dh), c4(dxs), N_s, c4(dxp), inv_row, idx, d_logit, c4(Ew), T, nvec, K,
        static_cast<uint4*>(du));
  return cuda_check(cudaGetLastError(), "unpermute_backward launch");
}

moe_status launch_unpermute_backward(const void* dh, const void* dx_shared, int N_s,
                                     const void* dx_perm, const int32_t* inv_row,
                                     const int32_t* idx, const float* d_logit, const void* E,
                                     moe_dtype dt, int T, int d, int K, void* du,
                                     cudaStream_t s) {
  const long long rb = (long long)d * (dt == MOE_F32 ? 4 : 2);
  if (gather_pipe_supported(GATHER_UNPERM_BWD, N_s, K, rb))
    return launch_gather_pipe(GATHER_UNPERM_BWD, dt, dh, nullptr, dx_shared, N_s, dx_perm,
                              (long long)T * K, E, inv_row, idx, d_logit, T, K, rb, du, nullptr,
                              nullptr, nullptr, s);
  if (dt == MOE_F32)
    return unpermute_bwd_dispatch<float>(dh, dx_shared, N_s, dx_perm, inv_row, idx, d_logit, E,
                                         T, d, K, du, s);
  return unpermute_bwd_dispatch<__nv_bfloat16>(dh, dx_shared, N_s, dx_perm, inv_row, idx,
                                               d_logit, E, T, d, K, du, s);
}

moe_status launch_router_weight_grad(const void* x_perm, const int32_t* x_rows,
                                     const float* d_logit_perm, const int32_t* offsets,
                                     moe_dtype dt, int N_r, int d, float* dE, cudaStream_t s) {
  const int per = dt == MOE_F32 ? 4 : 8;
  const int nvec = d / per;
  dim3 grid(N_r, (nvec + 127) / 128), block(128);
  if (dt == MOE_F32)
    router_weight_grad_kernel<float><<<grid, block, 0, s>>>(
        static_cast<const uint4*>(x_perm), x_rows, d_logit_perm, offsets, nvec, dE);
  else
    router_weight_grad_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        static_cast<const uint4*>(x_perm), x_rows, d_logit_perm, offsets, nvec, dE);
  return cuda_check(cudaGetLastError(), "router_weight_grad launch");
}

}  // namespace moe
