// Per-token steps of the layer backward: the gradient of the h'-equation
// through the combine, the gate normalisation and the affinity of
// "DeepSeek-V3 技術報告" (section 方法 / 2), and the unpermute that sums the
// input gradient (both run on the row-gather pipeline of gather.cu), and the
// centroid gradient.  The selection is held fixed (it is piecewise constant
// in s + b); gradients reach s only through g = s_sel / sum(s_sel).
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

moe_status launch_combine_backward(const void* dh, const void* u, const void* E,
                                   const void* y_perm, const int32_t* inv_row,
                                   const int32_t* idx, const float* gate, moe_dtype dt, int T,
                                   int d, int K, int N_r, void* dy_perm, float* d_gate,
                                   float* d_logit, float* d_logit_perm, cudaStream_t s) {
  const long long rb = (long long)d * (dt == MOE_F32 ? 4 : 2);
  return launch_gather_pipe(GATHER_COMBINE_BWD, dt, dh, u, nullptr, 0, y_perm, (long long)T * K,
                            E, N_r, inv_row, idx, gate, T, K, rb, dy_perm, d_gate, d_logit,
                            d_logit_perm, s);
}

moe_status launch_unpermute_backward(const void* dh, const void* dx_shared, int N_s,
                                     const void* dx_perm, const int32_t* inv_row,
                                     const int32_t* idx, const float* d_logit, const void* E,
                                     moe_dtype dt, int T, int d, int K, int N_r, void* du,
                                     cudaStream_t s) {
  const long long rb = (long long)d * (dt == MOE_F32 ? 4 : 2);
  return launch_gather_pipe(GATHER_UNPERM_BWD, dt, dh, nullptr, dx_shared, N_s, dx_perm,
                            (long long)T * K, E, N_r, inv_row, idx, d_logit, T, K, rb, du,
                            nullptr, nullptr, nullptr, s);
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
