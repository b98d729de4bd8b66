// Expert-parallel dispatch and return (the cross-device all-to-all of
// "DeepSeek V3 & R1 論文研究", sections DeepSeekMoE and Cross-Node
// All-to-All: routed experts are spread over devices, each token's rows go to
// the devices of its experts and the expert outputs come back).
//
// W ranks, N_r experts, E_loc = N_r / W experts per rank (expert e lives on
// rank e / E_loc).  C[s][e] = rows of source rank s routed to expert e (the
// all-gathered per-rank loads).  Rank d's receive buffer is grouped by its
// local expert j, inside by source rank, inside by the source's token order:
//   recv_off[d][j]  = sum_{j' < j} sum_s C[s][d E_loc + j']
//   base[d][j][s]   = recv_off[d][j] + sum_{s' < s} C[s'][d E_loc + j]
// Source rank s sends row (t, k) of expert e to rank d = e / E_loc at
//   base[d][e % E_loc][s] + (inv_row_s[t, k] - offsets_s[e])
// i.e. in the order its own permutation gives that expert's rows, and tags
// it with (s, inv_row_s[t, k]) so the expert output can be written back to
// the source's grouped position; the source then combines exactly as on one
// device.  Rows move with 16-byte stores straight into the destination
// buffers (peer memory over NVLink when the pointers are another GPU's).
#include "launch.h"

namespace moe {

namespace {

constexpr int kMaxRanks = 8;

struct RankPtrs {
  void* p[kMaxRanks];
};

// One block: per destination rank, a running sum over its experts.
__global__ void __launch_bounds__(kMaxRanks) ep_plan_kernel(const int32_t* __restrict__ C, int W,
                                                            int rank, int N_r,
                                                            int32_t* __restrict__ recv_offsets,
                                                            int32_t* __restrict__ send_base) {
  const int d = threadIdx.x;
  if (d >= W) return;
  const int E_loc = N_r / W;
  int run = 0;
  for (int j = 0; j < E_loc; ++j) {
    const int e = d * E_loc + j;
    if (d == rank) recv_offsets[j] = run;
    int before = 0;   // rows of this expert from ranks before `rank`
    int tot = 0;
    for (int s = 0; s < W; ++s) {
      const int c = C[(size_t)s * N_r + e];
      if (s < rank) before += c;
      tot += c;
    }
    send_base[e] = run + before;
    run += tot;
  }
  if (d == rank) recv_offsets[E_loc] = run;
}

// One warp per token: the row is read once and written to the K destinations.
template <int KMAX>
__global__ void __launch_bounds__(256) ep_dispatch_kernel(
    const uint4* __restrict__ u, int T, int nvec, int K, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ inv_row, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ send_base, int E_loc, int rank, RankPtrs rows, RankPtrs src,
    long long recv_cap, int* err) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  uint4* dst[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    dst[k] = nullptr;
    if (k < K) {
      const int e = idx[(size_t)t * K + k];
      const int r = inv_row[(size_t)t * K + k];
      const int dd = e / E_loc;
      const long long pos = (long long)send_base[e] + (r - offsets[e]);
      if (pos < 0 || pos >= recv_cap) {   // inconsistent loads: never write past a buffer
        if (lane == 0) atomicOr(err, ERR_EP_BOUNDS);
        continue;
      }
      dst[k] = static_cast<uint4*>(rows.p[dd]) + (size_t)pos * nvec;
      if (lane == 0) {
        int2* tag = static_cast<int2*>(src.p[dd]) + pos;
        *tag = make_int2(rank, r);
      }
    }
  }
  for (int c = lane; c < nvec; c += 32) {
    const uint4 v = u[(size_t)t * nvec + c];
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
      if (dst[k]) dst[k][c] = v;
  }
}

// One warp per received row: y goes back to (source rank, grouped position).
__global__ void __launch_bounds__(256) ep_return_kernel(const uint4* __restrict__ y,
                                                        const int2* __restrict__ tags,
                                                        const int32_t* __restrict__ n_rows,
                                                        int rows_cap, int nvec, int W,
                                                        RankPtrs ret, long long ret_cap,
                                                        int* err) {
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= *n_rows || p >= rows_cap) return;
  const int2 tag = tags[p];
  if (tag.x < 0 || tag.x >= W || tag.y < 0 || tag.y >= ret_cap) {
    if (lane == 0) atomicOr(err, ERR_EP_BOUNDS);
    return;
  }
  uint4* dst = static_cast<uint4*>(ret.p[tag.x]) + (size_t)tag.y * nvec;
  for (int c = lane; c < nvec; c += 32) dst[c] = y[(size_t)p * nvec + c];
}

}  // namespace

moe_status launch_ep_plan(const int32_t* counts_all, int W, int rank, int N_r,
                          int32_t* recv_offsets, int32_t* send_base, cudaStream_t s) {
  ep_plan_kernel<<<1, kMaxRanks, 0, s>>>(counts_all, W, rank, N_r, recv_offsets, send_base);
  return cuda_check(cudaGetLastError(), "ep_plan launch");
}

moe_status launch_ep_dispatch(const void* u, int elem_bytes, int T, int d, int K,
                              const int32_t* idx, const int32_t* inv_row, const int32_t* offsets,
                              const int32_t* send_base, int N_r, int W, int rank,
                              void* const* recv_rows, void* const* recv_src, long long recv_cap,
                              cudaStream_t s) {
  int* err = device_error_word();
  if (!err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  RankPtrs rows{}, src{};
  for (int i = 0; i < W; ++i) {
    rows.p[i] = recv_rows[i];
    src.p[i] = recv_src[i];
  }
  const int nvec = (int)((size_t)d * elem_bytes / 16);
  const int wpb = 8;
  dim3 grid((T + wpb - 1) / wpb), block(wpb * 32);
  auto U = static_cast<const uint4*>(u);
  if (K <= 8)
    ep_dispatch_kernel<8><<<grid, block, 0, s>>>(U, T, nvec, K, idx, inv_row, offsets, send_base,
                                                 N_r / W, rank, rows, src, recv_cap, err);
  else
    ep_dispatch_kernel<16><<<grid, block, 0, s>>>(U, T, nvec, K, idx, inv_row, offsets, send_base,
                                                  N_r / W, rank, rows, src, recv_cap, err);
  return cuda_check(cudaGetLastError(), "ep_dispatch launch");
}

moe_status launch_ep_return(const void* y, int elem_bytes, const void* recv_src,
                            const int32_t* n_rows, int rows_cap, int d, int W,
                            void* const* ret_rows, long long ret_cap, cudaStream_t s) {
  if (rows_cap <= 0) return MOE_OK;
  int* err = device_error_word();
  if (!err) return fail(MOE_ERR_CUDA, "device error word unavailable");
  RankPtrs ret{};
  for (int i = 0; i < W; ++i) ret.p[i] = ret_rows[i];
  const int nvec = (int)((size_t)d * elem_bytes / 16);
  const int wpb = 8;
  dim3 grid((rows_cap + wpb - 1) / wpb), block(wpb * 32);
  ep_return_kernel<<<grid, block, 0, s>>>(static_cast<const uint4*>(y),
                                          static_cast<const int2*>(recv_src), n_rows, rows_cap,
                                          nvec, W, ret, ret_cap, err);
  return cuda_check(cudaGetLastError(), "ep_return launch");
}

}  // namespace moe
