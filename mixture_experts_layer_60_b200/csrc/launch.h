// Internal launchers behind the C ABI (include/moe.h).  Every launcher
// assumes its arguments were validated by the entry point in api.cu.
#pragma once

#include "common.cuh"

namespace moe {

// router.cu ------------------------------------------------------------------
// logits[t, i] = sum_k u[t,k] E[i,k] on CUDA cores (float32 accumulation).
moe_status launch_logits_simt(const void* u, const void* E, moe_dtype dt, int T, int d,
                              int N_r, float* logits, cudaStream_t s);
// Float64 tie-break lists (device, inside the router workspace):
//   hdr[0]  tokens listed, hdr[1] candidate pairs (both zeroed before top-K)
//   tok, start, num [T]   per listed token: its id, first pair, number of pairs
//   pair [T*N_r]          candidate (token, expert) as t*N_r + e, grouped per token
struct RefineLists {
  int32_t* hdr;
  int32_t* tok;
  int32_t* start;
  int32_t* num;
  int32_t* pair;
};
// A token whose selection or output order was decided by a key gap below the
// refine gap is listed with every expert whose float32 key lies within the
// near distance of the lowest key a decision hinged on; the tie-break
// recomputes those experts' affinities in float64.  With B a bound on the
// float32 key error |s32 + b - (s64 + b)| of the tensor-core logits, a gap of
// 2B lists every token whose float32 selection or order can differ from the
// exact one, and a near distance of 2B or more recomputes every expert that
// can take part in it; the defaults are 2B and 3B.
constexpr float kRouterKeyErrorBound = 2e-5f;
constexpr float kRouterRefineGap = 2.0f * kRouterKeyErrorBound;
constexpr float kRouterNearBoundary = 3.0f * kRouterKeyErrorBound;
// The thresholds in force (moe_set_router_tie_break; defaults above).
void router_tie_break(float* refine_gap, float* near);
// sigmoid, biased top-K, gates, histogram (counts must be zeroed beforehand).
// n_groups > 1 && topk_groups < n_groups restricts each token to its best groups.
// A token whose routing was decided by a key gap < refine_gap is listed with
// the experts whose float32 key lies near one of its decision boundaries.
moe_status launch_topk(const float* logits, const float* b, int T, int N_r, int K, int n_groups,
                       int topk_groups, int32_t* idx, float* gate, int32_t* counts,
                       RefineLists rl, float refine_gap, float near, cudaStream_t s);

// router_tc.cu ----------------------------------------------------------------
// The fused router (logits on tcgen05 CTA pairs, sigmoid, biased top-K, gates,
// load, near-tie listing) for bf16 u and E with 32 <= N_r <= 256, N_r % 32 == 0,
// K <= 16 and, under a group limit, groups of a power-of-two size.  Writes the
// float32 logits rows of listed tokens only; counts must be zeroed and the
// tie-break header cleared beforehand.
bool router_tc_supported(moe_dtype dt, int d, int N_r, int K, int n_groups, int topk_groups);
moe_status launch_router_tc(const void* u, const void* E, const float* b, int T, int d, int N_r,
                            int K, int n_groups, int topk_groups, int32_t* idx, float* gate,
                            int32_t* counts, float* logits, RefineLists rl, float refine_gap,
                            float near, cudaStream_t s);
// Per listed token: float64 affinities of its listed experts, then its
// routing redone from them.
moe_status launch_refine(const void* u, const void* E, moe_dtype dt, const float* logits,
                         const float* b, int d, int N_r, int K, int n_groups, int topk_groups,
                         RefineLists rl, float near, int T, int32_t* idx, float* gate,
                         int32_t* counts, cudaStream_t s);

// permute.cu -----------------------------------------------------------------
size_t permute_ws_bytes(int T, int N_r);
// Argument checks shared by moe_permute and moe_permute_noalloc (api.cu);
// on success *elem_bytes is the size of one element of a row.
moe_status validate_permute_args(const char* who, const void* u, const float* u_scale,
                                 moe_dtype dt, const int32_t* topk_idx, int T, int d, int N_r,
                                 int K, const void* x_perm, const float* x_scale,
                                 const int32_t* offsets, const int32_t* perm_src,
                                 const int32_t* inv_row, int* elem_bytes);
// x_perm == nullptr: the grouping only (offsets, perm_src, inv_row), no rows copied.
moe_status launch_permute(const void* u, const float* u_scale, int elem_bytes, const int32_t* idx,
                          int T, int d, int N_r, int K, void* x_perm, float* x_scale,
                          int32_t* offsets, int32_t* perm_src, int32_t* inv_row,
                          void* ws, cudaStream_t s);

// ffn_simt.cu ----------------------------------------------------------------
// Grouped C[r, :] = epilogue(A[r, :] . B[g]^T) on CUDA cores.  swiglu: B has
// 2N rows (gate rows [0,N), up rows [N,2N)); C = SiLU(gate) * up.
// offsets == nullptr means one group covering all rows.
moe_status launch_simt_gemm(const void* A, const void* B, long long b_group_stride,
                            const int32_t* offsets, int n_groups, int rows, int N, int K,
                            bool swiglu, moe_dtype in_dt, void* C, moe_dtype out_dt,
                            cudaStream_t s);

// gemm_tc.cu -----------------------------------------------------------------
// Grouped bf16 GEMM on tcgen05 tensor cores (TMA -> smem -> tcgen05.mma -> TMEM).
enum TcEpilogue { TC_EPI_STORE_BF16 = 0, TC_EPI_STORE_F32 = 1, TC_EPI_SWIGLU_BF16 = 2 };
moe_status launch_tc_gemm(const void* A, const void* B, int b_rows_per_group,
                          const int32_t* offsets, int n_groups, int rows, int N, int K,
                          TcEpilogue epi, void* C, cudaStream_t s);

// gemm_ws.cu -----------------------------------------------------------------
// Weights-stationary grouped bf16 GEMM (expert FFNs): weights on the MMA's M
// side, each expert's tokens on N (tiles of <= 256 tokens, 16-row granularity).
// swiglu: B holds W_gate rows [0, I) and W_up rows [I, 2I) of a group.
// Extra groups (shared experts) run in the same launch: n_extra groups of T
// rows, weights W (row block j for group j), output rows rows + j*T of C;
// x_local: they read rows [0, T) of X (else their own C rows of the main X).
struct WsExtraGroups {
  const void* X = nullptr;
  const void* W = nullptr;
  int n_extra = 0;
  int T = 0;
  bool x_local = false;
};
moe_status launch_ws_gemm(const void* X, const void* W, int b_rows_per_group,
                          const int32_t* offsets, int n_groups, int rows, int N, int K,
                          bool swiglu, void* C, cudaStream_t s,
                          const WsExtraGroups* extra = nullptr);
// The STORE epilogue on CTA pairs (256 weight rows per pair, token tiles in
// multiples of 16, two TMEM accumulators per CTA, 128-wide K stages);
// launch_ws_gemm takes this path for the down projection whenever
// ws2_gemm_supported holds (N % 256 == 0, K % 128 == 0).
bool ws2_gemm_supported(int N, int K, int n_groups, bool grouped);
moe_status launch_ws2_gemm(const void* X, const void* W, int b_rows_per_group,
                           const int32_t* offsets, int n_groups, int rows, int N, int K, void* C,
                           cudaStream_t s, const WsExtraGroups* extra = nullptr);
// Epilogues: SWIGLU  C = SiLU(gate) * up (N = I columns);
//            SWIGLU_SAVE  the same, plus S[:, 0:I] = gate, S[:, I:2I] = up;
//            STORE   C = the product (N columns);
//            DSWIGLU dh = the product (N = I columns), a = S[:, 0:I], b = S[:, I:2I]:
//                    C[:, 0:I] = dh * b * SiLU'(a), C[:, I:2I] = dh * SiLU(a).
// w_mn: W is stored [G*K rows][N cols] (N contiguous) instead of [G*rows_per_group][K].
enum WsEpi { WS_SWIGLU = 0, WS_STORE = 1, WS_SWIGLU_SAVE = 2, WS_DSWIGLU = 3 };
moe_status launch_ws_gemm_ex(const void* X, const void* W, int b_rows_per_group,
                             const int32_t* offsets, int n_groups, int rows, int N, int K,
                             WsEpi epi, bool w_mn, void* C, int ldc, void* S, int lds,
                             cudaStream_t s, const WsExtraGroups* extra = nullptr);

// gather.cu ------------------------------------------------------------------
// Row-gather pipeline (bulk copies into a shared-memory ring, four producer
// warps, four consumer warps) for the per-token combine kernels.
enum GatherMode { GATHER_COMBINE = 0, GATHER_COMBINE_BWD = 1, GATHER_UNPERM_BWD = 2 };
// Supported when K <= 16 and the row slots of a job (COMBINE 1 + N_s + K,
// COMBINE_BWD 2 + 2K, UNPERM_BWD 1 + N_s + 2K) are at most 64.
bool gather_pipe_supported(int mode, int N_s, int K, long long row_bytes);
// a: u (COMBINE) or dh; b: u (COMBINE_BWD); sh: shared-expert rows [N_s][T];
// perm: grouped rows (n_perm of them); cent: centroids [N_r] (backward);
// w: gate or d_logit.  Slots with a grouped row outside [0, n_perm) or
// (backward) an expert id outside [0, N_r) are left out.
moe_status launch_gather_pipe(int mode, moe_dtype dt, const void* a, const void* b,
                              const void* sh, int N_s, const void* perm, long long n_perm,
                              const void* cent, int N_r, const int32_t* inv_row,
                              const int32_t* idx, const float* w, int T, int K,
                              long long row_bytes, void* out, float* d_gate, float* d_logit,
                              float* d_logit_perm, cudaStream_t s);

// gemm_wgrad.cu --------------------------------------------------------------
// C[g] [M, N] = sum over the rows r of group g of A[r, :]^T B[r, :] (bf16 in and out).
// A_tail: scratch of wgrad_tail_bytes(M * 2, 64, groups) bytes for the groups'
// zero-padded last 64-row blocks of A.
moe_status launch_wgrad_gemm(const void* A, int M, const void* B, int N, const int32_t* offsets,
                             int n_groups, int rows, void* A_tail, void* C, cudaStream_t s);
// T[g] = the last block_rows-row block of group g of A (rows past the group zeroed).
moe_status launch_wgrad_tails(const void* A, size_t row_bytes, int block_rows,
                              const int32_t* offsets, int n_groups, int rows, void* T,
                              cudaStream_t s);
size_t wgrad_tail_bytes(size_t row_bytes, int block_rows, int n_groups);

// gemm_wgrad_fp8.cu ----------------------------------------------------------
// C[g] [M, N] = sum over g's 128-row blocks b of (qa_b^T qb_b) * sa[b, m] * sb[b, n].
// qa_tail: scratch of wgrad_tail_bytes(M, 128, groups) bytes.
moe_status launch_wgrad_fp8(const void* qa, const float* sa, int M, const void* qb,
                            const float* sb, int N, const int32_t* offsets, int n_groups,
                            int rows, const int32_t* block_start, void* qa_tail, void* C,
                            cudaStream_t s);

// gemm_fp8.cu ----------------------------------------------------------------
moe_status launch_fp8_gemm(const void* A, const float* a_scale, const void* B,
                           const float* b_scale, int b_rows_per_group,
                           const int32_t* offsets, int n_groups, int rows, int N, int K,
                           bool swiglu, void* C, float* c_scale, cudaStream_t s);
// Epilogues as in gemm_fp8.cu's header; b_mn: B stored [G*K rows][N cols].
enum Fp8Epi { F8_SWIGLU = 0, F8_STORE = 1, F8_SWIGLU_SAVE = 2, F8_DSWIGLU = 3 };
moe_status launch_fp8_gemm_ex(const void* A, const float* a_scale, const void* B,
                              const float* b_scale, int b_rows_per_group, const int32_t* offsets,
                              int n_groups, int rows, int N, int K, Fp8Epi epi, bool b_mn,
                              void* C, float* c_scale, void* S, int lds, void* C2,
                              cudaStream_t s);
moe_status launch_quant_1x128(const void* x, int rows, int cols, uint8_t* q, float* scale,
                              cudaStream_t s);
moe_status launch_quant_128x128(const void* w, int groups, int rows, int cols, uint8_t* q,
                                float* scale, cudaStream_t s);
// Wgrad operands: group-aligned 128-row blocks, one scale per (block, column).
// block_start[g] = first block of group g (computed by launch_block_table).
moe_status launch_block_table(const int32_t* offsets, int n_groups, int rows,
                              int32_t* block_start, cudaStream_t s);
// x [*, ldx] bf16; row r of the operand is x[src_rows ? src_rows[r] : r];
// swiglu_in: the operand is SiLU(x[:, 0:cols]) * x[:, cols:2cols].
// q [rows, cols] e4m3, scale [blocks, cols] float32.
moe_status launch_quant_128x1(const void* x, int ldx, const int32_t* src_rows, bool swiglu_in,
                              int rows, int cols, const int32_t* offsets, int n_groups,
                              const int32_t* block_start, uint8_t* q, float* scale,
                              cudaStream_t s);

// combine.cu -----------------------------------------------------------------
moe_status launch_combine(const void* u, const void* y_shared, int N_s, const void* y_perm,
                          const int32_t* inv_row, const float* gate, moe_dtype dt, int T,
                          int d, int K, void* h_out, cudaStream_t s);
moe_status launch_bias_update(float* b, const int32_t* counts, int N_r, int T, int K,
                              float gamma, cudaStream_t s);

// backward.cu ----------------------------------------------------------------
moe_status launch_combine_backward(const void* dh, const void* u, const void* E,
                                   const void* y_perm, const int32_t* inv_row,
                                   const int32_t* idx, const float* gate, moe_dtype dt, int T,
                                   int d, int K, int N_r, void* dy_perm, float* d_gate,
                                   float* d_logit, float* d_logit_perm, cudaStream_t s);
moe_status launch_unpermute_backward(const void* dh, const void* dx_shared, int N_s,
                                     const void* dx_perm, const int32_t* inv_row,
                                     const int32_t* idx, const float* d_logit, const void* E,
                                     moe_dtype dt, int T, int d, int K, int N_r, void* du,
                                     cudaStream_t s);
moe_status launch_router_weight_grad(const void* x, const int32_t* x_rows,
                                     const float* d_logit_perm, const int32_t* offsets,
                                     moe_dtype dt, int N_r, int d, float* dE, cudaStream_t s);

// ep.cu ----------------------------------------------------------------------
// Expert-parallel receive layout, dispatch and return (see ep.cu's header).
moe_status launch_ep_plan(const int32_t* counts_all, int W, int rank, int N_r,
                          int32_t* recv_offsets, int32_t* send_base, cudaStream_t s);
moe_status launch_ep_dispatch(const void* u, int elem_bytes, int T, int d, int K,
                              const int32_t* idx, const int32_t* inv_row, const int32_t* offsets,
                              const int32_t* send_base, int N_r, int W, int rank,
                              void* const* recv_rows, void* const* recv_src, long long recv_cap,
                              cudaStream_t s);
moe_status launch_ep_return(const void* y, int elem_bytes, const void* recv_src,
                            const int32_t* n_rows, int rows_cap, int d, int W,
                            void* const* ret_rows, long long ret_cap, cudaStream_t s);

}  // namespace moe
