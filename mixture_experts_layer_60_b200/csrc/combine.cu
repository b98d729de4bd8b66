// Combine with the residual, the h'-equation of "DeepSeek-V3 技術報告"
// (section 方法 / 2):
//   h'_t = u_t + sum_j FFN^(s)_j(u_t) + sum_k g_{t,k} FFN^(r)_{idx(t,k)}(u_t),
// and the per-step bias rule of the same section.
#include "launch.h"

namespace moe {

// One warp per token; each lane walks the row in 16-byte vectors.  Every
// input row is read exactly once; sums are float32 in the order
// u, shared experts (j ascending), routed experts (slot k ascending).
template <typename E, int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ u,
                                                      const uint4* __restrict__ ys, int N_s,
                                                      const uint4* __restrict__ yp,
                                                      const int32_t* __restrict__ inv_row,
                                                      const float* __restrict__ gate, int T,
                                                      int nvec, int K, uint4* __restrict__ out) {
  constexpr int N = Vec<E>::N;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int rows[KMAX];
  float g[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    if (k < K) {
      rows[k] = inv_row[(size_t)t * K + k];
      g[k] = gate[(size_t)t * K + k];
    }
  }
  for (int c = lane; c < nvec; c += 32) {
    float acc[N], tmp[N];
    Vec<E>::load(u[(size_t)t * nvec + c], acc);
    for (int j = 0; j < N_s; ++j) {
      Vec<E>::load(ys[((size_t)j * T + t) * nvec + c], tmp);
#pragma unroll
      for (int i = 0; i < N; ++i) acc[i] += tmp[i];
    }
    uint4 raw[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
      if (k < K) raw[k] = yp[(size_t)rows[k] * nvec + c];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K) {
        Vec<E>::load(raw[k], tmp);
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = fmaf(g[k], tmp[i], acc[i]);
      }
    }
    out[(size_t)t * nvec + c] = Vec<E>::store(acc);
  }
}

// Generic K (> 16): slots read one after another.
template <typename E>
__global__ void __launch_bounds__(256) combine_kernel_anyk(const uint4* __restrict__ u,
                                                           const uint4* __restrict__ ys, int N_s,
                                                           const uint4* __restrict__ yp,
                                                           const int32_t* __restrict__ inv_row,
                                                           const float* __restrict__ gate, int T,
                                                           int nvec, int K,
                                                           uint4* __restrict__ out) {
  constexpr int N = Vec<E>::N;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  for (int c = lane; c < nvec; c += 32) {
    float acc[N], tmp[N];
    Vec<E>::load(u[(size_t)t * nvec + c], acc);
    for (int j = 0; j < N_s; ++j) {
      Vec<E>::load(ys[((size_t)j * T + t) * nvec + c], tmp);
      for (int i = 0; i < N; ++i) acc[i] += tmp[i];
    }
    for (int k = 0; k < K; ++k) {
      const float gk = gate[(size_t)t * K + k];
      Vec<E>::load(yp[(size_t)inv_row[(size_t)t * K + k] * nvec + c], tmp);
      for (int i = 0; i < N; ++i) acc[i] = fmaf(gk, tmp[i], acc[i]);
    }
    out[(size_t)t * nvec + c] = Vec<E>::store(acc);
  }
}

template <typename E>
static void combine_dispatch(const void* u, const void* ys, int N_s, const void* yp,
                             const int32_t* inv_row, const float* gate, int T, int d, int K,
                             void* out, cudaStream_t s) {
  const int nvec = d / Vec<E>::N;
  const int wpb = 8;
  dim3 grid((T + wpb - 1) / wpb), block(wpb * 32);
  auto U = static_cast<const uint4*>(u);
  auto YS = static_cast<const uint4*>(ys);
  auto YP = static_cast<const uint4*>(yp);
  auto O = static_cast<uint4*>(out);
  if (K <= 8)
    combine_kernel<E, 8><<<grid, block, 0, s>>>(U, YS, N_s, YP, inv_row, gate, T, nvec, K, O);
  else if (K <= 16)
    combine_kernel<E, 16><<<grid, block, 0, s>>>(U, YS, N_s, YP, inv_row, gate, T, nvec, K, O);
  else
    combine_kernel_anyk<E><<<grid, block, 0, s>>>(U, YS, N_s, YP, inv_row, gate, T, nvec, K, O);
}

moe_status launch_combine(const void* u, const void* y_shared, int N_s, const void* y_perm,
                          const int32_t* inv_row, const float* gate, moe_dtype dt, int T,
                          int d, int K, void* h_out, cudaStream_t s) {
  const long long rb = (long long)d * (dt == MOE_F32 ? 4 : 2);
  if (gather_pipe_supported(GATHER_COMBINE, N_s, K, rb))
    return launch_gather_pipe(GATHER_COMBINE, dt, u, nullptr, y_shared, N_s, y_perm,
                              (long long)T * K, nullptr, 0, inv_row, nullptr, gate, T, K, rb,
                              h_out, nullptr, nullptr, nullptr, s);
  if (dt == MOE_F32)
    combine_dispatch<float>(u, y_shared, N_s, y_perm, inv_row, gate, T, d, K, h_out, s);
  else
    combine_dispatch<__nv_bfloat16>(u, y_shared, N_s, y_perm, inv_row, gate, T, d, K, h_out, s);
  return cuda_check(cudaGetLastError(), "combine launch");
}

// Bias rule: compare the load with the mean T*K/N_r in integers
// (counts*N_r vs T*K) so that the mean need not be representable.
__global__ void bias_update_kernel(float* __restrict__ b, const int32_t* __restrict__ counts,
                                   int N_r, long long TK, float gamma) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N_r) return;
  const long long load = (long long)counts[i] * N_r;
  if (load > TK) b[i] = b[i] - gamma;
  else if (load < TK) b[i] = b[i] + gamma;
}

moe_status launch_bias_update(float* b, const int32_t* counts, int N_r, int T, int K,
                              float gamma, cudaStream_t s) {
  bias_update_kernel<<<(N_r + 255) / 256, 256, 0, s>>>(b, counts, N_r, (long long)T * K, gamma);
  return cuda_check(cudaGetLastError(), "bias_update launch");
}

}  // namespace moe
