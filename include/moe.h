/*
 * moe.h - C ABI of the B200 DeepSeekMoE layer library (libmoe.so).
 *
 * The layer is the one defined in "DeepSeek-V3 技術報告" (xyznot.com summary
 * of arXiv 2412.19437), section 方法 / 2 "具備無輔助損失平衡機制的 DeepSeekMoE":
 *
 *   s_{i,t} = Sigmoid(u_t^T e_i)                               (affinity)
 *   g'_{i,t} = s_{i,t} if s_{i,t} + b_i in Topk({s_{j,t} + b_j}, K), else 0
 *   g_{i,t}  = g'_{i,t} / sum_j g'_{j,t}                        (normalised)
 *   h'_t = u_t + sum_{j<N_s} FFN^(s)_j(u_t) + sum_i g_{i,t} FFN^(r)_i(u_t)
 *   b_i <- b_i - gamma if expert i is overloaded, + gamma if underloaded
 *
 * with FFN(x) = W_down (SiLU(W_gate x) * (W_up x)), and, optionally, the FP8
 * recipe of the same page's section 核心概念 (E4M3, 1x128 activation tiles,
 * 128x128 weight blocks, FP32 promotion every 128 K-elements).
 *
 * Conventions shared by every call
 *   - Pointers named as device buffers are CUDA device pointers on the current
 *     device; the caller owns every buffer.  Scratch space, where a call needs
 *     any, is the caller's `workspace`, sized by the matching *_workspace_size().
 *   - Arrays are row-major and contiguous.  bf16 is IEEE bfloat16, e4m3 is the
 *     OCP FP8 E4M3 ("fn") byte format.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns; none synchronises the host, except
 *     moe_device_status().
 *   - Arguments are checked before anything is launched; a bad argument
 *     returns a status and launches nothing.  No call aborts, traps or prints.
 *     moe_last_error() describes the last failure on the calling thread.
 *   - Kernels run on sm_100a (B200) only; other devices get MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, non-positive or inconsistent size */
  MOE_ERR_UNSUPPORTED = 2,   /* dtype/shape combination or device not supported */
  MOE_ERR_WORKSPACE = 3,     /* workspace smaller than *_workspace_size() */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call or a launch failed */
  MOE_ERR_TIMEOUT = 5        /* a kernel gave up a bounded wait (see moe_device_status) */
} moe_status;

typedef enum moe_dtype {
  MOE_F32 = 0,
  MOE_BF16 = 1,
  MOE_E4M3 = 2
} moe_dtype;

/* Version of this ABI (increments on any signature change). */
int moe_abi_version(void);

/* Text of the last error on the calling thread ("" if none).  Static storage
 * owned by the library; valid until the next failing call on this thread. */
const char* moe_last_error(void);

/* Name of a status code. */
const char* moe_status_string(moe_status status);

/* ------------------------------------------------------------------------
 * moe_route - affinity, biased top-K, gate normalisation and load histogram
 * (affinity line and g'-equation of section 2).
 *
 *   u        [T, d]    device, dt (MOE_F32 or MOE_BF16): token states u_t
 *   E        [N_r, d]  device, dt: expert centroids e_i
 *   b        [N_r]     device, float32: routing bias (steers selection only)
 *   topk_idx [T, K]    device, int32 out: selected experts, largest s+b first,
 *                      lower index first on equal keys
 *   topk_gate[T, K]    device, float32 out: g = s / (sum of the selected s),
 *                      from the unbiased s
 *   counts   [N_r]     device, int32 out: number of tokens routed to each
 *                      expert (overwritten, not accumulated)
 *   workspace          device, >= moe_route_workspace_size(T, N_r) bytes
 * Logits are accumulated in float32 from the stored values; sigmoid, keys and
 * gates are float32.  Tokens whose selection (or output order) was decided by
 * a key gap below the refine gap (default 4e-5) are re-routed from float64
 * logits for every expert within the near distance (default 6e-5) of the
 * boundary (sigmoid in float64, s rounded once to float32), so the float32
 * accumulation error cannot flip them; the defaults are 2B and 3B for the
 * key-error bound B = 2e-5 of the tensor-core logits (see
 * moe_set_router_tie_break).  Requires 1 <= K <= N_r <= 1024, d % 64 == 0 and
 * rows of at most 32 KB (d <= 16384 bf16, 8192 float32).
 * ------------------------------------------------------------------------ */
size_t moe_route_workspace_size(int T, int N_r);

/* moe_set_router_tie_break - the thresholds of the float64 tie-break of
 * moe_route / moe_route_grouped: a token is re-routed when a key gap that
 * decided its selection or output order is below refine_gap, from float64
 * affinities of every expert whose float32 key lies within `near` of the
 * lowest key a decision hinged on.  Both >= 0; (0, 0) restores the defaults
 * (4e-5, 6e-5).  Values below the defaults give up the exactness guarantee;
 * larger values re-route more tokens (a refine gap of, say, 1e30 re-routes
 * every token and leaves every token's float32 logit row in the first
 * T*N_r floats of the workspace).  Process-wide, from the next call on. */
moe_status moe_set_router_tie_break(float refine_gap, float near);

moe_status moe_route(const void* u, const void* E, moe_dtype dt, const float* b,
                     int T, int d, int N_r, int K,
                     int32_t* topk_idx, float* topk_gate, int32_t* counts,
                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_route_grouped - moe_route with a group limit: experts form n_groups
 * groups of N_r/n_groups consecutive indices and each token may only select
 * experts of its topk_groups best groups (the per-token node limit of
 * "DeepSeek V3 & R1 論文研究", section Cross-Node All-to-All, which gives
 * only the limit).  A group's score is its largest key s+b (this library's
 * reading); ties keep the lower group index.  Same arguments, outputs and
 * workspace as moe_route, plus
 *   n_groups     1..32, dividing N_r
 *   topk_groups  1..n_groups, with topk_groups * N_r/n_groups >= K
 * moe_route is moe_route_grouped with n_groups = topk_groups = 1.
 * ------------------------------------------------------------------------ */
moe_status moe_route_grouped(const void* u, const void* E, moe_dtype dt, const float* b,
                             int T, int d, int N_r, int K, int n_groups, int topk_groups,
                             int32_t* topk_idx, float* topk_gate, int32_t* counts,
                             void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_permute - group the T*K (token, slot) pairs by expert and copy the
 * token rows into that order (the dispatch step that feeds FFN^(r)_i in the
 * h'-equation).  Inside an expert's group tokens keep ascending order.
 *
 *   u        [T, d]      device, dt (MOE_F32, MOE_BF16 or MOE_E4M3)
 *   u_scale  [T, d/128]  device, float32: only for MOE_E4M3 (tile scales of u), else NULL
 *   topk_idx [T, K]      device, int32: from moe_route (an id outside [0, N_r)
 *                        is left out: its inv_row is -1 and no row is copied)
 *   x_perm   [T*K, d]    device, dt out: x_perm[p] = u[perm_src[p]]
 *   x_scale  [T*K, d/128] device, float32 out (MOE_E4M3 only, else NULL)
 *   offsets  [N_r+1]     device, int32 out: group g is rows [offsets[g], offsets[g+1])
 *   perm_src [T*K]       device, int32 out: grouped row -> token
 *   inv_row  [T, K]      device, int32 out: (token, slot) -> grouped row
 *   workspace            device, >= moe_permute_workspace_size(T, N_r) bytes
 * Requires d * sizeof(dt) % 16 == 0 and 1 <= K <= N_r <= 1024.
 * ------------------------------------------------------------------------ */
size_t moe_permute_workspace_size(int T, int N_r);
moe_status moe_permute(const void* u, const float* u_scale, moe_dtype dt,
                       const int32_t* topk_idx, int T, int d, int N_r, int K,
                       void* x_perm, float* x_scale,
                       int32_t* offsets, int32_t* perm_src, int32_t* inv_row,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_permute_index - the grouping of moe_permute without the row copies:
 * offsets, perm_src and inv_row exactly as moe_permute writes them, for
 * callers that move the token rows themselves (the expert-parallel dispatch,
 * moe_ep_dispatch, reads them from u through inv_row).  Same requirements on
 * topk_idx, T, N_r, K and the workspace (>= moe_permute_workspace_size(T,
 * N_r) bytes).
 * ------------------------------------------------------------------------ */
moe_status moe_permute_index(const int32_t* topk_idx, int T, int N_r, int K, int32_t* offsets,
                             int32_t* perm_src, int32_t* inv_row, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_expert_ffn - grouped SwiGLU expert FFN: for every group g and every row
 * r in [offsets[g], offsets[g+1]):
 *     y[r] = W_down[g] (SiLU(W_gate[g] x[r]) * (W_up[g] x[r]))
 * (FFN_i of the h'-equation; the SwiGLU form is this library's reading).
 *
 *   x          [rows, d]        device, dt
 *   x_scale    [rows, d/128]    device, float32 (MOE_E4M3 only, else NULL)
 *   offsets    [n_groups+1]     device, int32, non-decreasing, offsets[0] = 0,
 *                               offsets[n_groups] <= rows.  Values outside
 *                               [0, rows], or below an earlier value, are
 *                               clamped on the device (bf16 / FP8: each raised
 *                               to the largest earlier value and cut to rows;
 *                               f32: each group's range cut into [0, rows));
 *                               rows outside every group are not written and
 *                               moe_device_status() reports bit 16
 *   W_gate_up  [n_groups, 2I, d] device, dt: rows [0,I) are W_gate, [I,2I) W_up
 *   w_scale_gate_up [n_groups, 2I/128, d/128] float32 (MOE_E4M3 only, else NULL)
 *   W_down     [n_groups, d, I] device, dt
 *   w_scale_down    [n_groups, d/128, I/128]  float32 (MOE_E4M3 only, else NULL)
 *   y          [rows, d]        device out: float32 for MOE_F32, bf16 otherwise.
 *                               Rows outside every group are not written.
 *   workspace                   device, >= moe_expert_ffn_workspace_size(dt, rows, I)
 * Arithmetic: MOE_F32 - float32 FMA; MOE_BF16 - tcgen05 tensor cores, float32
 * accumulation in TMEM, SwiGLU in float32, the intermediate rounded to bf16;
 * MOE_E4M3 - each 128-wide K block's partial sum is promoted to float32 with
 * its activation and weight scales, the intermediate is re-quantised 1x128.
 * Requires d % 128 == 0 and I % 128 == 0.
 * ------------------------------------------------------------------------ */
size_t moe_expert_ffn_workspace_size(moe_dtype dt, int rows, int I);
moe_status moe_expert_ffn(const void* x, const float* x_scale, const int32_t* offsets,
                          int n_groups, int rows, int d, int I, moe_dtype dt,
                          const void* W_gate_up, const float* w_scale_gate_up,
                          const void* W_down, const float* w_scale_down,
                          void* y, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_expert_gate_up / moe_expert_down - the two halves of moe_expert_ffn,
 * for callers that schedule or time them apart (same layouts and rules):
 *   gate_up: h[r] = SiLU(W_gate[g] x[r]) * (W_up[g] x[r])
 *            h [rows, I]: float32 (MOE_F32), bf16 (MOE_BF16) or e4m3 with
 *            h_scale [rows, I/128] float32 (MOE_E4M3; h_scale NULL otherwise)
 *   down:    y[r] = W_down[g] h[r]
 * moe_expert_ffn(...) is gate_up into its workspace followed by down.
 * ------------------------------------------------------------------------ */
moe_status moe_expert_gate_up(const void* x, const float* x_scale, const int32_t* offsets,
                              int n_groups, int rows, int d, int I, moe_dtype dt,
                              const void* W_gate_up, const float* w_scale_gate_up,
                              void* h, float* h_scale, void* stream);
moe_status moe_expert_down(const void* h, const float* h_scale, const int32_t* offsets,
                           int n_groups, int rows, int d, int I, moe_dtype dt,
                           const void* W_down, const float* w_scale_down, void* y, void* stream);

/* ------------------------------------------------------------------------
 * moe_expert_gate_up_shared / moe_expert_down_shared - the two halves of the
 * routed grouped FFN with the N_s shared experts of the h'-equation (every
 * token, weight 1) run as extra groups of the same launch, so that their
 * tiles fill the routed launch's tail.  MOE_BF16 only; same arithmetic as
 * moe_expert_gate_up / moe_expert_down.
 *   x          [rows, d]        device bf16: routed rows (moe_permute's x_perm)
 *   offsets    [n_groups+1]     device int32: routed groups, as moe_expert_ffn
 *   u          [T, d]           device bf16: the layer input (shared experts' rows)
 *   W_gate_up  [n_groups, 2I, d], Ws_gate_up [N_s, 2I, d]   device bf16
 *   W_down     [n_groups, d, I],  Ws_down    [N_s, d, I]    device bf16
 *   h          [rows + N_s*T, I] device bf16: routed rows first, then shared
 *              expert j's rows at rows + j*T + t (SiLU(gate) * up of u[t])
 *   y          [rows + N_s*T, d] device bf16: y[r] = W_down[g] h[r] for the
 *              routed rows, y[rows + j*T + t] = Ws_down[j] h[rows + j*T + t];
 *              so y + rows*d is the y_shared [N_s, T, d] of moe_combine.
 * Requires d % 256 == 0 and I % 128 == 0 (down: d a multiple of 256).
 * ------------------------------------------------------------------------ */
moe_status moe_expert_gate_up_shared(const void* x, const int32_t* offsets, int n_groups,
                                     int rows, const void* u, int T, int N_s, int d, int I,
                                     const void* W_gate_up, const void* Ws_gate_up, void* h,
                                     void* stream);
moe_status moe_expert_down_shared(const void* h, const int32_t* offsets, int n_groups, int rows,
                                  int T, int N_s, int d, int I, const void* W_down,
                                  const void* Ws_down, void* y, void* stream);

/* ------------------------------------------------------------------------
 * moe_combine - the h'-equation with the residual:
 *   h_out[t] = u[t] + sum_{j<N_s} y_shared[j][t] + sum_k topk_gate[t,k] y_perm[inv_row[t,k]]
 * summed in float32, rounded once to dt.
 *
 *   u         [T, d]       device, dt (MOE_F32 or MOE_BF16)
 *   y_shared  [N_s, T, d]  device, dt (may be NULL when N_s == 0)
 *   y_perm    [T*K, d]     device, dt: routed expert outputs in grouped order
 *   inv_row   [T, K]       device, int32: from moe_permute (a slot outside
 *                          [0, T*K), e.g. -1, adds nothing)
 *   topk_gate [T, K]       device, float32: from moe_route
 *   h_out     [T, d]       device, dt out (must not alias the inputs)
 * Requires d * sizeof(dt) % 16 == 0.
 * ------------------------------------------------------------------------ */
moe_status moe_combine(const void* u, const void* y_shared, int N_s,
                       const void* y_perm, const int32_t* inv_row, const float* topk_gate,
                       moe_dtype dt, int T, int d, int K, void* h_out, void* stream);

/* ------------------------------------------------------------------------
 * moe_bias_update - the bias rule of section 2: with the mean load T*K/N_r,
 *   b_i <- b_i - gamma  if counts_i * N_r > T * K   (overloaded)
 *   b_i <- b_i + gamma  if counts_i * N_r < T * K   (underloaded)
 *   b_i unchanged       if equal                    (gamma = 0.001 on the page)
 * float32 arithmetic, in place.  counts from moe_route (or their sum over
 * data-parallel replicas, with T the replicas' total token count).
 * ------------------------------------------------------------------------ */
moe_status moe_bias_update(float* b, const int32_t* counts, int N_r, int T, int K,
                           float gamma, void* stream);

/* ------------------------------------------------------------------------
 * FP8 quantisers (recipe of section 核心概念, FP8 bullet).  scale = amax/448
 * in float32 (1 for an all-zero tile); q = E4M3_rne_satfinite(x / scale) with
 * an IEEE float32 division.
 *
 * moe_quantize_1x128: x [rows, cols] bf16 -> q [rows, cols] e4m3,
 *                     scale [rows, cols/128] float32.  cols % 128 == 0.
 * moe_quantize_128x128: w [groups, rows, cols] bf16 -> q e4m3,
 *                     scale [groups, rows/128, cols/128] float32.
 *                     rows % 128 == 0, cols % 128 == 0.
 * ------------------------------------------------------------------------ */
moe_status moe_quantize_1x128(const void* x, int rows, int cols,
                              uint8_t* q, float* scale, void* stream);
moe_status moe_quantize_128x128(const void* w, int groups, int rows, int cols,
                                uint8_t* q, float* scale, void* stream);

/* ------------------------------------------------------------------------
 * moe_permute_noalloc - moe_permute for callers that cannot allocate device
 * memory.  The DeepSeek-V3 pages have no counterpart; it exists for callers
 * that run inside a host framework which owns every device allocation (a
 * caching allocator or fixed arena it does not expose) or in loops that must
 * not allocate once started, and so cannot pass a workspace.
 *
 * Same arguments, layouts and results as moe_permute, without the workspace.
 * Its scratch is a static 1 MiB device array inside the library (held by
 * every GPU that loads libmoe.so until the process exits), so it accepts
 * only 2 * ceil(T/256) * N_r * 4 bytes <= 1 MiB (T <= 131072 at N_r = 256);
 * larger problems get MOE_ERR_UNSUPPORTED and launch nothing.  The first
 * call on a device looks up the array's device address (make it before any
 * stream capture) and keeps it for the life of the process: a
 * cudaDeviceReset unloads the array, so do not use the library across one.
 * Every call uses the same array: calls whose work overlaps on the GPU
 * (other streams or host threads) race on it.
 * ------------------------------------------------------------------------ */
moe_status moe_permute_noalloc(const void* u, const float* u_scale, moe_dtype dt,
                               const int32_t* topk_idx, int T, int d, int N_r, int K,
                               void* x_perm, float* x_scale,
                               int32_t* offsets, int32_t* perm_src, int32_t* inv_row,
                               void* stream);

/* ========================================================================
 * Layer backward.  "DeepSeek V3 & R1 論文研究", section FP8 mixed precision,
 * names the three GEMM passes of training (Fprop, Dgrad for activations,
 * Wgrad for weights) and keeps the MoE gating module in its original
 * precision; the pages print no backward formulas, so these calls apply the
 * chain rule to the forward of section 方法 / 2 of "DeepSeek-V3 技術報告".
 * The selection (top-K of s + b) is piecewise constant and is held fixed:
 * gradients reach s only through g = s_sel / sum(s_sel); b gets none.
 * Expert GEMMs run in bf16 with float32 accumulation (MOE_BF16) or under the
 * FP8 recipe (MOE_E4M3); d % 256 == 0 and I % 256 == 0.  Order of a training
 * step:
 *   forward:  moe_route, moe_permute, moe_expert_gate_up_save (routed and
 *             shared), moe_expert_down, moe_combine
 *   backward: moe_combine_backward, moe_expert_ffn_backward (routed with
 *             dy_perm, shared with dh_out), moe_unpermute_backward,
 *             moe_router_weight_grad
 * ======================================================================== */

/* ------------------------------------------------------------------------
 * moe_expert_gate_up_save - moe_expert_gate_up (MOE_BF16 or MOE_E4M3, same
 * arguments and outputs) that also keeps the pre-activations the backward
 * needs, computed in float32 and stored bf16:
 *   a_gu[r, 0:I]  = W_gate[g] x[r],  a_gu[r, I:2I] = W_up[g] x[r]
 *   h[r]          = SiLU(gate) * up from the float32 values (bf16, or e4m3
 *                   with h_scale for MOE_E4M3)
 *   a_gu [rows, 2I] device bf16 out, 16-byte aligned.
 * ------------------------------------------------------------------------ */
moe_status moe_expert_gate_up_save(const void* x, const float* x_scale, const int32_t* offsets,
                                   int n_groups, int rows, int d, int I, moe_dtype dt,
                                   const void* W_gate_up, const float* w_scale_gate_up, void* h,
                                   float* h_scale, void* a_gu, void* stream);

/* ------------------------------------------------------------------------
 * moe_combine_backward - gradient of the h'-equation through the routed
 * term, the gate normalisation and the affinity, for upstream dh_out = dL/dh':
 *   dy_perm[inv_row[t,k]]      = topk_gate[t,k] * dh_out[t]       (dt)
 *   d_gate[t,k]                = <dh_out[t], y_perm[inv_row[t,k]]>  (float32)
 *   s_k = Sigmoid(u[t] . E[topk_idx[t,k]]) recomputed in float32, S = sum_k s_k
 *   d_logit[t,k]               = (d_gate[t,k] - sum_j topk_gate[t,j] d_gate[t,j]) / S
 *                                * s_k (1 - s_k)                    (float32)
 *   d_logit_perm[inv_row[t,k]] = d_logit[t,k]                      (float32)
 *   dh_out, u [T, d]; E [N_r, d]; y_perm [T*K, d]: device, dt (MOE_F32 or
 *   MOE_BF16); inv_row, topk_idx [T, K] int32 and topk_gate [T, K] float32
 *   from the forward; dy_perm [T*K, d] dt out; d_gate, d_logit [T, K] and
 *   d_logit_perm [T*K] float32 out.  N_r: rows of E.  K <= 16,
 *   d * sizeof(dt) % 16 == 0.
 *   A slot whose inv_row lies outside [0, T*K) or whose expert id lies
 *   outside [0, N_r) (moe_permute gives such ids inv_row -1) is left out of
 *   the selection: no dy_perm row is written, no d_logit_perm entry, its
 *   d_gate and d_logit are 0, its s is not part of S, and neither its row
 *   nor its centroid is read.
 * The shared experts' upstream gradient is dh_out itself (weight 1).
 * ------------------------------------------------------------------------ */
moe_status moe_combine_backward(const void* dh_out, const void* u, const void* E,
                                const void* y_perm, const int32_t* inv_row,
                                const int32_t* topk_idx, const float* topk_gate, moe_dtype dt,
                                int T, int d, int K, int N_r, void* dy_perm, float* d_gate,
                                float* d_logit, float* d_logit_perm, void* stream);

/* ------------------------------------------------------------------------
 * moe_quantize_128x1_grouped - FP8 quantiser of a weight-gradient operand
 * (reading of the 1x128 activation tile for a contraction over an expert's
 * tokens): blocks of 128 consecutive rows start at every group's first row
 * (the last block of a group may be shorter; empty groups have none), and
 * each column of a block gets scale = amax/448 (1 if all zero);
 * q = E4M3_rne_satfinite(x / scale) with an IEEE float32 division.
 *   x            [rows, cols] device bf16, cols % 128 == 0
 *   offsets      [n_groups+1] device int32 (NULL: one group of all rows)
 *   q            [rows, cols] device e4m3 out
 *   scale        [ceil(rows/128) + n_groups, cols] device float32 out; row
 *                block_start[g] + i holds block i of group g
 *   block_start  [n_groups+1] device int32 out: first block of each group,
 *                block_start[n_groups] = number of blocks
 * ------------------------------------------------------------------------ */
moe_status moe_quantize_128x1_grouped(const void* x, int rows, int cols, const int32_t* offsets,
                                      int n_groups, uint8_t* q, float* scale,
                                      int32_t* block_start, void* stream);

/* ------------------------------------------------------------------------
 * moe_expert_ffn_backward - Dgrad and Wgrad of the grouped SwiGLU FFN for
 * upstream dy.  For group g and its rows r, with a, b the gate and up halves
 * of a_gu and h = SiLU(a) * b from moe_expert_gate_up_save:
 *   dh  = dy W_down[g]                               (float32, not stored)
 *   dA  = [dh * b * SiLU'(a) | dh * SiLU(a)]          (in the workspace)
 *   dx[r]          = dA[r] W_gate_up[g]               (Dgrad, bf16)
 *   dW_down[g]     = sum_r dy[r]^T h[r]               (Wgrad, [d, I] bf16)
 *   dW_gate_up[g]  = sum_r dA[r]^T x[r]               (Wgrad, [2I, d] bf16)
 * MOE_BF16: bf16 GEMMs with float32 accumulation; x [rows, d] and h
 *   [rows, I] bf16, x_rows and the weight scales NULL.
 * MOE_E4M3: every GEMM input E4M3 (the FP8 recipe applied to Dgrad and
 *   Wgrad): dy and dA quantised per row and 128 columns for the two Dgrads;
 *   for the Wgrads dy, h, dA and x quantised per column and 128 consecutive
 *   rows of one group (blocks start at the group's first row); weights
 *   W_gate_up / W_down e4m3 with their forward 128x128 block scales
 *   (w_scale_gate_up [n_groups, 2I/128, d/128], w_scale_down
 *   [n_groups, d/128, I/128]); each 128-deep partial sum promoted with its
 *   two scales.  x is the bf16 layer input: row r is x[x_rows[r]] when
 *   x_rows (device int32 [rows]) is given, else x[r]; h may be NULL (it is
 *   recomputed from a_gu).
 *   x [*, d], dy [rows, d], a_gu [rows, 2I]: device bf16 in; offsets
 *   [n_groups+1] as for moe_expert_ffn; dx [rows, d], dW_gate_up and dW_down
 *   (same shapes as the weights) device bf16 out.  A group with no rows gets
 *   zero weight gradients.  Workspace: moe_expert_ffn_backward_workspace_size
 *   bytes (it depends on n_groups for MOE_E4M3), 256-byte aligned.
 *   d % 256 == 0, I % 256 == 0.
 * ------------------------------------------------------------------------ */
size_t moe_expert_ffn_backward_workspace_size(moe_dtype dt, int rows, int d, int I,
                                              int n_groups);
moe_status moe_expert_ffn_backward(const void* x, const int32_t* x_rows, const int32_t* offsets,
                                   int n_groups, int rows, int d, int I, moe_dtype dt,
                                   const void* W_gate_up, const float* w_scale_gate_up,
                                   const void* W_down, const float* w_scale_down,
                                   const void* a_gu, const void* h, const void* dy, void* dx,
                                   void* dW_gate_up, void* dW_down, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_unpermute_backward - the input gradient:
 *   du[t] = dh_out[t] + sum_{j<N_s} dx_shared[j][t] + sum_k dx_perm[inv_row[t,k]]
 *           + sum_k d_logit[t,k] E[topk_idx[t,k]]
 * summed in float32 in that order, rounded once to dt.  dh_out, du [T, d];
 * dx_shared [N_s, T, d] (NULL when N_s == 0); dx_perm [T*K, d]; E [N_r, d]:
 * device, dt (MOE_F32 or MOE_BF16); N_r rows of E.  K <= 16, N_s + 2K <= 63,
 * d * sizeof(dt) % 16 == 0.  A slot whose inv_row lies outside [0, T*K) or
 * whose expert id lies outside [0, N_r) is left out of both sums (neither
 * its dx_perm row nor its centroid is read).
 * ------------------------------------------------------------------------ */
moe_status moe_unpermute_backward(const void* dh_out, const void* dx_shared, int N_s,
                                  const void* dx_perm, const int32_t* inv_row,
                                  const int32_t* topk_idx, const float* d_logit, const void* E,
                                  moe_dtype dt, int T, int d, int K, int N_r, void* du,
                                  void* stream);

/* ------------------------------------------------------------------------
 * moe_router_weight_grad - gradient of the expert centroids E:
 *   dE[i] = sum over grouped rows r of expert i of d_logit_perm[r] x(r)
 * with x(r) = x[x_rows[r]] when x_rows is given (e.g. u and perm_src from
 * moe_permute), else x[r] (x_perm); rows in ascending order, float32
 * accumulation.  x device dt (MOE_F32 or MOE_BF16), d_logit_perm [rows]
 * float32 and offsets [N_r+1] from moe_combine_backward / moe_permute;
 * dE [N_r, d] device float32 out (original precision for the gating
 * module).  d * sizeof(dt) % 16 == 0.
 * ------------------------------------------------------------------------ */
moe_status moe_router_weight_grad(const void* x, const int32_t* x_rows,
                                  const float* d_logit_perm, const int32_t* offsets,
                                  moe_dtype dt, int N_r, int d, float* dE, void* stream);

/* ========================================================================
 * Expert parallelism ("DeepSeek V3 & R1 論文研究", sections DeepSeekMoE and
 * Cross-Node All-to-All: routed experts spread over devices, tokens sent to
 * the devices of their experts and the outputs returned).  W ranks (W <= 8,
 * N_r % W == 0), E_loc = N_r / W experts per rank, expert e on rank e/E_loc.
 * counts_all [W, N_r] int32: every rank's per-expert load (moe_route counts,
 * all-gathered).  Rank d receives its rows grouped by local expert j,
 * inside by source rank, inside by the source's token order:
 *   recv_offsets[j] = sum_{j'<j} sum_s counts_all[s][d*E_loc + j']
 * so the local grouped FFN runs on (recv_rows, recv_offsets, E_loc groups).
 * A step on rank s: moe_route, moe_permute (for offsets / inv_row),
 * moe_ep_plan, moe_ep_dispatch, [every rank's rows have arrived],
 * moe_expert_ffn on the received rows, moe_ep_return, [every rank's outputs
 * have arrived], moe_combine with y_perm = the return buffer.  The result
 * equals the single-device layer's bit for bit.  Destination pointers may
 * be another GPU's memory (peer access, e.g. symmetric memory); the calls
 * only store to them.  Row positions outside a buffer's capacity are never
 * written: the row is skipped and moe_device_status reports it.
 * ======================================================================== */

/* moe_ep_plan - this rank's receive offsets recv_offsets [E_loc+1] and, for
 * every expert e, send_base [N_r]: where this rank's first row of expert e
 * lands in the receive buffer of rank e/E_loc.  counts_all device int32. */
moe_status moe_ep_plan(const int32_t* counts_all, int W, int rank, int N_r,
                       int32_t* recv_offsets, int32_t* send_base, void* stream);

/* moe_ep_dispatch - sends row (t, k) of u (this rank's tokens [T, d], dt
 * MOE_F32 or MOE_BF16) to rank d = topk_idx[t,k]/E_loc, at position
 * send_base[e] + inv_row[t,k] - offsets[e] of recv_rows[d] ([recv_cap, d]
 * rows of dt), and writes the tag (rank, inv_row[t,k]) at the same position
 * of recv_tags[d] ([recv_cap] x int32 pairs).  recv_rows / recv_tags: host
 * arrays of W device pointers.  topk_idx, inv_row, offsets: this rank's
 * moe_route / moe_permute outputs. */
moe_status moe_ep_dispatch(const void* u, moe_dtype dt, int T, int d, int K,
                           const int32_t* topk_idx, const int32_t* inv_row,
                           const int32_t* offsets, const int32_t* send_base, int N_r, int W,
                           int rank, void* const* recv_rows, void* const* recv_tags,
                           long long recv_cap, void* stream);

/* moe_ep_return - writes row p of y ([recv_cap, d] dt, the expert outputs of
 * the received rows; p < recv_offsets[E_loc]) to row tag.y of ret_rows[tag.x]
 * ([ret_cap, d] dt on every rank: its grouped positions), tag = recv_tags[p].
 * n_rows: device pointer to the received row count (recv_offsets + E_loc). */
moe_status moe_ep_return(const void* y, moe_dtype dt, const void* recv_tags,
                         const int32_t* n_rows, long long recv_cap, int d, int W,
                         void* const* ret_rows, long long ret_cap, void* stream);

/* ------------------------------------------------------------------------
 * moe_device_status - synchronises the current device, then returns (and
 * clears) the library's device-side error word: 0 if no kernel gave up a
 * bounded wait or clamped bad input since the last call, else a bit set
 * naming the kernel:
 *   1  a tcgen05 bf16 GEMM (expert FFN, router logits, Wgrad)
 *   2  an FP8 tcgen05 GEMM
 *   4  an expert-parallel copy skipped a row position past its buffer
 *   8  the row-gather pipeline (combine, combine and unpermute backward)
 *  16  a grouped GEMM met group offsets outside [0, rows] or decreasing and
 *      clamped them (no row outside [0, rows) was read or written)
 *  32  (bounds-checked build libmoe_checked.so only, compiled with
 *      -DMOE_CHECK_BOUNDS) an internal index lay outside the buffer it
 *      addresses; the access was skipped
 * ------------------------------------------------------------------------ */
moe_status moe_device_status(int* flags);

/* ------------------------------------------------------------------------
 * moe_set_pipeline_wait_limit - the bound, in nanoseconds, of every wait of
 * the row-gather pipeline (moe_combine, moe_combine_backward,
 * moe_unpermute_backward) on a shared-memory stage; 0 restores the default
 * of 1 s.  After a wait runs out the kernel stops taking rows, lets the
 * copies it issued land (within 1 s), returns, and moe_device_status()
 * reports bit 8; rows it did not reach are not written.  Process-wide; it
 * takes effect at the next launch.  The pages have no counterpart: the
 * knob exists so that the timeout path can be exercised.
 * ------------------------------------------------------------------------ */
moe_status moe_set_pipeline_wait_limit(unsigned long long ns);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
