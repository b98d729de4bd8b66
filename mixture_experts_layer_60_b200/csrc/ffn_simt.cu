// CUDA-core grouped GEMM with an optional SwiGLU epilogue.  It serves the
// float32 configuration (tensor cores would round the operands) and the
// float32 router logits.  Per group g and row r in [offsets[g], offsets[g+1]):
//   C[r, n] = sum_k A[r, k] B_g[n, k]                       (plain)
//   C[r, n] = SiLU(sum_k A[r,k] B_g[n,k]) * sum_k A[r,k] B_g[N+n,k]   (swiglu)
// 64x64 output tile per 256-thread block, 4x4 outputs per thread, K step 16.
#include <math.h>

#include "launch.h"

namespace moe {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename Tin, typename Tout, bool SWIGLU>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const Tin* __restrict__ A,
                                                        const Tin* __restrict__ B,
                                                        long long b_group_stride,
                                                        const int32_t* __restrict__ offsets,
                                                        int n_groups, int rows, int N, int K,
                                                        Tout* __restrict__ C) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Us[SWIGLU ? BK : 1][BN + 4];
  __shared__ int s_group, s_mtile;

  // Map blockIdx.y to (group, m-tile of that group).
  if (threadIdx.x == 0) {
    int g = -1, mt = 0;
    if (offsets == nullptr) {
      if ((long long)blockIdx.y * BM < rows) { g = 0; mt = blockIdx.y; }
    } else {
      int acc = 0;
      for (int i = 0; i < n_groups; ++i) {
        int r0, r1;
        clamp_group_rows(offsets, i, rows, nullptr, r0, r1);
        const int m = r1 - r0;
        const int tiles = (m + BM - 1) / BM;
        if ((int)blockIdx.y < acc + tiles) { g = i; mt = blockIdx.y - acc; break; }
        acc += tiles;
      }
    }
    s_group = g;
    s_mtile = mt;
  }
  __syncthreads();
  const int g = s_group;
  if (g < 0) return;
  int row0, row_end;
  clamp_group_rows(offsets, g, rows, nullptr, row0, row_end);
  const int m0 = row0 + s_mtile * BM;
  const int n0 = blockIdx.x * BN;
  const Tin* Bg = B + (long long)g * b_group_stride;

  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {}, accu[4][4] = {};

  for (int k0 = 0; k0 < K; k0 += BK) {
    // A tile: 64 rows x 16 k, 4 elements per thread
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      const int gr = m0 + r;
      As[kk][r] = (gr < row_end && k0 + kk < K) ? IO<Tin>::cvt(A[(size_t)gr * K + k0 + kk]) : 0.f;
    }
    for (int i = threadIdx.x; i < BN * BK; i += 256) {
      const int n = i / BK, kk = i % BK;
      const int gn = n0 + n;
      const bool ok = gn < N && k0 + kk < K;
      Bs[kk][n] = ok ? IO<Tin>::cvt(Bg[(size_t)gn * K + k0 + kk]) : 0.f;
      if (SWIGLU) Us[kk][n] = ok ? IO<Tin>::cvt(Bg[(size_t)(N + gn) * K + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], bb[4], uu[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bb[j] = Bs[kk][tx * 4 + j];
        if (SWIGLU) uu[j] = Us[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
          if (SWIGLU) accu[i][j] = fmaf(a[i], uu[j], accu[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (SWIGLU) v = (v / (1.0f + expf(-v))) * accu[i][j];
      C[(size_t)r * N + n] = IO<Tout>::to(v);
    }
  }
}

template <typename Tin, typename Tout>
void simt_launch(const void* A, const void* B, long long bstride, const int32_t* offsets,
                 int n_groups, int rows, int N, int K, bool swiglu, void* C, cudaStream_t s) {
  const int mtiles = (rows + BM - 1) / BM + (offsets ? n_groups : 0);
  dim3 grid((N + BN - 1) / BN, mtiles > 0 ? mtiles : 1);
  if (swiglu)
    simt_gemm_kernel<Tin, Tout, true><<<grid, 256, 0, s>>>(
        (const Tin*)A, (const Tin*)B, bstride, offsets, n_groups, rows, N, K, (Tout*)C);
  else
    simt_gemm_kernel<Tin, Tout, false><<<grid, 256, 0, s>>>(
        (const Tin*)A, (const Tin*)B, bstride, offsets, n_groups, rows, N, K, (Tout*)C);
}

}  // namespace

moe_status launch_simt_gemm(const void* A, const void* B, long long b_group_stride,
                            const int32_t* offsets, int n_groups, int rows, int N, int K,
                            bool swiglu, moe_dtype in_dt, void* C, moe_dtype out_dt,
                            cudaStream_t s) {
  if (in_dt == MOE_F32 && out_dt == MOE_F32)
    simt_launch<float, float>(A, B, b_group_stride, offsets, n_groups, rows, N, K, swiglu, C, s);
  else if (in_dt == MOE_BF16 && out_dt == MOE_F32)
    simt_launch<__nv_bfloat16, float>(A, B, b_group_stride, offsets, n_groups, rows, N, K, swiglu,
                                      C, s);
  else if (in_dt == MOE_BF16 && out_dt == MOE_BF16)
    simt_launch<__nv_bfloat16, __nv_bfloat16>(A, B, b_group_stride, offsets, n_groups, rows, N, K,
                                              swiglu, C, s);
  else
    return fail(MOE_ERR_UNSUPPORTED, "simt gemm: unsupported dtype pair");
  return cuda_check(cudaGetLastError(), "simt_gemm launch");
}

}  // namespace moe
