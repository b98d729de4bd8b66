"""CPU oracle for the DeepSeekMoE layer forward (TEST INFRASTRUCTURE ONLY).

This module is the plain, slow, obviously-correct reference that the CUDA
library is checked against.  Only the test-suite, the smoke check and the
CPU-baseline leg of the benchmark may import it; the library itself never
does, and nothing here is shared with the CUDA sources.

Source of every formula: "DeepSeek-V3 技術報告" (xyznot.com summary of
arXiv 2412.19437), section 方法 / 2. "具備無輔助損失平衡機制的 DeepSeekMoE":

  * h'-equation  : h'_t = u_t + sum_s FFN_s(u_t) + sum_i g_{i,t} FFN_i(u_t)
  * affinity     : s_{i,t} = Sigmoid(u_t^T e_i)
  * g'-equation  : g'_{i,t} = s_{i,t} if s_{i,t}+b_i is in Topk({s_{j,t}+b_j}, K_r), else 0;
                   g is g' normalised
  * bias rule    : overloaded expert -> b_i - gamma, underloaded -> b_i + gamma, gamma = 0.001
  * FP8 recipe   : same page, section 核心概念, "FP8 混合精度訓練" bullet: E4M3 everywhere,
                   1x128 activation tiles, 128x128 weight blocks, FP32 promotion every
                   N_c = 128 accumulation steps.

Readings taken where the page is silent:

  R1  g = g' / sum_j g'_j over the selected experts (no extra scale, no epsilon; s > 0).
  R2  top-K ties go to the lower expert index; the K outputs are ordered by
      descending biased key, lower index first on equal keys.
  R3  gating arithmetic: logits from the stored values in float64, sigmoid in
      float64, s rounded once to float32; s + b and the top-K compare in float32
      (the precision the kernels take that decision in).
  R4  "overloaded" / "underloaded" compare the expert's load with the mean load
      T*K/N_r, in integers (counts*N_r vs T*K); equal load leaves b unchanged.
  R5  FFN_i is SwiGLU: W_down (SiLU(W_gate x) * (W_up x)), SiLU(z) = z / (1 + e^-z);
      shared experts have the same width I as routed ones and weight 1.
  R11 group limit (optional): a group's score is its largest s+b; keep the
      topk_groups best groups (ties to the lower group index), select top-K
      inside them.  The pages give only the limit (at most 4 nodes per token).
  R6  FP8: E4M3 max 448, round-to-nearest-even, saturate to +-448; a tile's
      scale is amax/448 in float32 (1 for an all-zero tile); q = E4M3(x / scale)
      with x / scale an IEEE float32 division; weights quantised per 128x128
      block, activations per 1x128 row tile, both FFN inputs (x and h) quantised;
      each 128-wide K block's partial sum is multiplied by s_a * s_w and added.
      h is formed in float32 before it is quantised.

Nothing here is blocked, fused or reordered beyond those definitions.
"""
from __future__ import annotations

import numpy as np

GAMMA = 0.001          # bias step (bias rule above)
E4M3_MAX = 448.0       # largest finite E4M3 magnitude (R6)
FP8_TILE = 128         # N_c and the tile edge of the FP8 recipe


# ----------------------------------------------------------------------------
# Router: affinity, biased top-K, gate normalisation, load
# ----------------------------------------------------------------------------

def affinity(u: np.ndarray, E: np.ndarray) -> np.ndarray:
    """s_{i,t} = Sigmoid(u_t^T e_i)  (affinity line of section 2; reading R3).

    u: [T, d], E: [N_r, d], both holding the exact stored values (any float
    dtype).  Returns s as float32 [T, N_r].
    """
    x = np.asarray(u, np.float64) @ np.asarray(E, np.float64).T
    s = 1.0 / (1.0 + np.exp(-x))
    return s.astype(np.float32)


def biased_topk(s: np.ndarray, b: np.ndarray, K: int):
    """Selection of the g'-equation: the K experts with the largest s + b.

    Keys are formed in float32 (R3).  A stable sort of the negated keys puts
    the largest key first and, among equal keys, the lower index first (R2).
    Returns (idx [T, K] int32, key [T, N_r] float32).
    """
    s = np.asarray(s, np.float32)
    key = (s + np.asarray(b, np.float32)[None, :]).astype(np.float32)
    order = np.argsort(-key, axis=1, kind="stable")
    return order[:, :K].astype(np.int32), key


def grouped_topk(s, b, K, n_groups, topk_groups):
    """Group-limited selection (the node limit of "DeepSeek V3 & R1 論文研究",
    section Cross-Node All-to-All: a token reaches at most a few nodes).
    Experts form n_groups groups of N_r/n_groups consecutive indices.  Reading
    R11: a group's score is its largest biased key s+b; the topk_groups groups
    with the largest scores are kept (ties to the lower group index), then the
    K largest keys among the kept groups' experts are selected exactly as in
    biased_topk.  Returns (idx [T, K] int32, key [T, N_r] float32)."""
    s = np.asarray(s, np.float32)
    key = (s + np.asarray(b, np.float32)[None, :]).astype(np.float32)
    T, N_r = key.shape
    gs = N_r // n_groups
    gscore = key.reshape(T, n_groups, gs).max(axis=2)
    gorder = np.argsort(-gscore, axis=1, kind="stable")[:, :topk_groups]
    keep = np.zeros((T, n_groups), bool)
    np.put_along_axis(keep, gorder, True, axis=1)
    masked = np.where(np.repeat(keep, gs, axis=1), key, -np.inf).astype(np.float32)
    order = np.argsort(-masked, axis=1, kind="stable")
    return order[:, :K].astype(np.int32), key


def route_grouped(u, E, b, K, n_groups, topk_groups):
    """Router with the group limit: as route(), selection by grouped_topk."""
    s = affinity(u, E)
    idx, key = grouped_topk(s, b, K, n_groups, topk_groups)
    return {"s": s, "key": key, "idx": idx, "gate": gates(s, idx),
            "counts": load_counts(idx, E.shape[0])}


def gates(s: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_{i,t} = g'_{i,t} / sum_j g'_{j,t}: the unbiased s of the selected
    experts, normalised to sum 1 (g'-equation + reading R1).  float32 out."""
    sel = np.take_along_axis(np.asarray(s, np.float32), idx, axis=1).astype(np.float64)
    return (sel / sel.sum(axis=1, keepdims=True)).astype(np.float32)


def load_counts(idx: np.ndarray, N_r: int) -> np.ndarray:
    """counts_i = number of (token, slot) pairs routed to expert i: the load
    the bias rule measures."""
    return np.bincount(np.asarray(idx).reshape(-1), minlength=N_r).astype(np.int32)


def route(u, E, b, K):
    """Router of section 2 for every token: returns a dict with
    s [T,N_r] f32, key [T,N_r] f32, idx [T,K] i32, gate [T,K] f32, counts [N_r] i32."""
    s = affinity(u, E)
    idx, key = biased_topk(s, b, K)
    return {"s": s, "key": key, "idx": idx, "gate": gates(s, idx),
            "counts": load_counts(idx, E.shape[0])}


def topk_margins(key: np.ndarray, idx: np.ndarray):
    """Per token: (gap between the K-th and (K+1)-th largest key, smallest gap
    between adjacent selected keys).  Used only to exempt near-ties when the
    GPU's routing is compared with this one."""
    srt = -np.sort(-key, axis=1)
    K = idx.shape[1]
    kth = srt[:, K - 1].astype(np.float64)
    nxt = srt[:, K].astype(np.float64) if key.shape[1] > K else np.full(key.shape[0], -np.inf)
    inner = (np.min(srt[:, :K - 1] - srt[:, 1:K], axis=1).astype(np.float64)
             if K > 1 else np.full(key.shape[0], np.inf))
    return kth - nxt, inner


# ----------------------------------------------------------------------------
# Permutation into per-expert groups
# ----------------------------------------------------------------------------

def permute_indices(idx: np.ndarray, N_r: int):
    """Group the T*K (token, slot) pairs by expert, tokens ascending inside a
    group (stable).  Returns offsets [N_r+1] (exclusive scan of the load),
    perm_src [T*K] (grouped row -> token) and inv_row [T, K] ((t, k) -> grouped row)."""
    T, K = idx.shape
    flat = np.asarray(idx, np.int64).reshape(-1)
    order = np.argsort(flat, kind="stable")          # by expert, then by t*K+k
    counts = np.bincount(flat, minlength=N_r)
    offsets = np.zeros(N_r + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    perm_src = (order // K).astype(np.int32)
    inv = np.empty(T * K, np.int64)
    inv[order] = np.arange(T * K)
    return offsets.astype(np.int32), perm_src, inv.reshape(T, K).astype(np.int32)


# ----------------------------------------------------------------------------
# Expert FFN (reading R5) and the layer (h'-equation)
# ----------------------------------------------------------------------------

def silu(z):
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(x, W_gate, W_up, W_down):
    """FFN(x) = W_down (SiLU(W_gate x) * (W_up x)), rows of x are tokens.
    W_gate, W_up: [I, d]; W_down: [d, I].  float64 throughout."""
    x = np.asarray(x, np.float64)
    g = x @ np.asarray(W_gate, np.float64).T
    v = x @ np.asarray(W_up, np.float64).T
    return (silu(g) * v) @ np.asarray(W_down, np.float64).T


def layer_forward(u, idx, gate, routed, shared):
    """h'_t = u_t + sum_s FFN_s(u_t) + sum_{i in S_t} g_{i,t} FFN_i(u_t)  (h'-equation).

    u: [T, d]; idx/gate: routing of these T tokens; routed[e] and shared[j]
    return (W_gate, W_up, W_down) as arrays (a list, or any object with
    __getitem__ that yields them lazily).  Evaluated expert by expert so each
    weight matrix is touched once.  float64 result [T, d].
    """
    u = np.asarray(u, np.float64)
    out = u.copy()
    for j in range(len(shared)):
        out += swiglu_ffn(u, *shared[j])
    idx = np.asarray(idx)
    for e in np.unique(idx):
        t, k = np.nonzero(idx == e)
        y = swiglu_ffn(u[t], *routed[int(e)])
        out[t] += np.asarray(gate, np.float64)[t, k][:, None] * y
    return out


# ----------------------------------------------------------------------------
# Bias update (bias rule + reading R4)
# ----------------------------------------------------------------------------

def bias_update(b, counts, T, K, gamma=GAMMA):
    """b_i - gamma if counts_i*N_r > T*K (overloaded), b_i + gamma if < (underloaded),
    unchanged if equal.  float32 arithmetic, as b is stored."""
    b = np.asarray(b, np.float32)
    c = np.asarray(counts, np.int64)
    N_r = b.shape[0]
    load, mean = c * N_r, int(T) * int(K)
    g = np.float32(gamma)
    out = b.copy()
    out[load > mean] = (b[load > mean] - g).astype(np.float32)
    out[load < mean] = (b[load < mean] + g).astype(np.float32)
    return out


# ----------------------------------------------------------------------------
# FP8 recipe (reading R6)
# ----------------------------------------------------------------------------

def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value (1 sign, 4 exponent bits with bias 7, 3 mantissa bits),
    ties to even, saturated to +-448.  Normal numbers have spacing 2^(e-3) in the
    binade [2^e, 2^(e+1)); below the smallest normal 2^-6 the spacing is 2^-9."""
    x = np.asarray(x, np.float64)
    _, ex = np.frexp(x)                       # |x| = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)                # binade exponent, clamped to the subnormal range
    quantum = np.ldexp(1.0, e - 3)
    q = np.round(x / quantum) * quantum       # np.round is round-half-to-even
    return np.clip(q, -E4M3_MAX, E4M3_MAX)


def tile_scale(amax) -> np.ndarray:
    """scale = amax / 448 in float32 (1 for an all-zero tile)."""
    amax = np.asarray(amax, np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(amax == 0, np.float32(1.0), s).astype(np.float32)


def quant_1x128(X):
    """Activation quantisation: one float32 scale per row and 128-column tile.
    X: [R, D] (D a multiple of 128).  Returns (q [R, D] float64 holding E4M3
    values, scale [R, D/128] float32)."""
    X = np.asarray(X, np.float32)
    R, D = X.shape
    t = X.reshape(R, D // FP8_TILE, FP8_TILE)
    sc = tile_scale(np.abs(t).max(axis=2))
    q = e4m3_round((t / sc[:, :, None]).astype(np.float32))
    return q.reshape(R, D), sc


def quant_128x128(W):
    """Weight quantisation: one float32 scale per 128x128 block.
    W: [N, K].  Returns (q [N, K] float64 E4M3 values, scale [N/128, K/128] float32)."""
    W = np.asarray(W, np.float32)
    N, K = W.shape
    t = W.reshape(N // FP8_TILE, FP8_TILE, K // FP8_TILE, FP8_TILE)
    sc = tile_scale(np.abs(t).max(axis=(1, 3)))
    q = e4m3_round((t / sc[:, None, :, None]).astype(np.float32))
    return q.reshape(N, K), sc


def fp8_promoted_gemm(qa, sa, qw, sw):
    """C[r, n] = sum over 128-wide K blocks kb of
         (sum_{k in kb} qa[r, k] qw[n, k]) * sa[r, kb] * sw[n // 128, kb]
    i.e. each N_c = 128 partial sum is promoted with its two scales.  float64."""
    qa = np.asarray(qa, np.float64)
    qw = np.asarray(qw, np.float64)
    R, Kd = qa.shape
    N = qw.shape[0]
    out = np.zeros((R, N), np.float64)
    rows_blk = np.arange(N) // FP8_TILE
    for kb in range(Kd // FP8_TILE):
        sl = slice(kb * FP8_TILE, (kb + 1) * FP8_TILE)
        part = qa[:, sl] @ qw[:, sl].T
        out += part * np.asarray(sa, np.float64)[:, kb][:, None] \
                    * np.asarray(sw, np.float64)[rows_blk, kb][None, :]
    return out


def fp8_swiglu_ffn(x, Wq):
    """SwiGLU FFN under the FP8 recipe.  x: [R, d] activations (exact stored
    values); Wq: dict with q/scale pairs 'gate', 'up', 'down' from quant_128x128.
    Steps: quantise x 1x128 -> promoted GEMMs -> SiLU(gate)*up in float64,
    rounded to float32 -> quantise h 1x128 -> promoted GEMM.  float64 result."""
    qx, sx = quant_1x128(x)
    g = fp8_promoted_gemm(qx, sx, *Wq["gate"])
    v = fp8_promoted_gemm(qx, sx, *Wq["up"])
    h = (silu(g) * v).astype(np.float32)
    qh, sh = quant_1x128(h)
    return fp8_promoted_gemm(qh, sh, *Wq["down"])


def quantise_expert(W_gate, W_up, W_down):
    """Offline 128x128 quantisation of one expert's three matrices."""
    return {"gate": quant_128x128(W_gate), "up": quant_128x128(W_up),
            "down": quant_128x128(W_down)}


def layer_forward_fp8(u, idx, gate, routed_q, shared_q):
    """h'-equation with every expert FFN evaluated under the FP8 recipe.
    routed_q[e] / shared_q[j] give quantise_expert(...) dicts.  The residual
    and the gate weights stay in the original precision."""
    u = np.asarray(u, np.float64)
    out = u.copy()
    for j in range(len(shared_q)):
        out += fp8_swiglu_ffn(u, shared_q[j])
    idx = np.asarray(idx)
    for e in np.unique(idx):
        t, k = np.nonzero(idx == e)
        y = fp8_swiglu_ffn(u[t], routed_q[int(e)])
        out[t] += np.asarray(gate, np.float64)[t, k][:, None] * y
    return out
