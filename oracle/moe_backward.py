"""CPU oracle for the DeepSeekMoE layer backward (TEST INFRASTRUCTURE ONLY).

Gradients of the layer of moe_oracle.layer_forward with respect to its input
u, the router's expert centroids E and every expert's W_gate, W_up, W_down,
for an upstream gradient dh = dL/dh'.  Only the test-suite may import this.

Source: "DeepSeek-V3 技術報告" (xyznot.com summary of arXiv 2412.19437),
section 方法 / 2 (h'-equation, affinity, g'-equation), and "DeepSeek V3 & R1
論文研究" section FP8 mixed precision, which names the three GEMM passes of
training: Fprop (forward), Dgrad (activation gradient) and Wgrad (weight
gradient), and keeps the MoE gating module in its original precision.  The
pages print no backward formulas; what follows is the chain rule applied to
the forward definitions, step by step in reverse order.

Readings taken where the pages are silent:

  B1  The selection S_t (top-K of s+b) is piecewise constant in u, E and b:
      it is held fixed and has no gradient; b receives none.  Gradient flows
      into s only through the gate values g = s_sel / sum(s_sel).
  B2  The backward is the derivative of the exact (float64) forward: s is not
      rounded to float32 here.
  B3  L = <dh, h'>: du collects the residual, the shared and routed expert
      paths and the router path.
  B5  FP8 backward (the recipe of section 核心概念 applied to Dgrad and Wgrad):
      every GEMM input is E4M3; an activation tile is 1 x 128 along the
      contraction, so Dgrad inputs (dy, dA) are quantised per row and 128
      columns, and Wgrad inputs (dy, h, dA, x: contraction over an expert's
      tokens) per column and 128 consecutive rows of one expert, the blocks
      starting at the expert's first row (the last block may be shorter).
      Weights keep their forward 128x128 blocks (square, so the transposed
      use needs no new scales).  Each 128-deep partial sum is promoted with
      its two scales.  The backward starts from the forward's float64 a, b
      (SiLU's inputs) and h = SiLU(a) * b rounded to float32; dA is rounded to
      float32 before it is quantised; gradients of the gate and the router
      stay in the original precision.

Everything is float64.  Nothing is fused or reordered beyond the definitions.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import (FP8_TILE, e4m3_round, fp8_promoted_gemm, fp8_swiglu_ffn, quant_1x128,
                         silu, swiglu_ffn, tile_scale)


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu_grad(z):
    """d/dz [z * sigmoid(z)] = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    sg = sigmoid(z)
    return sg * (1.0 + z * (1.0 - sg))


def swiglu_ffn_backward(x, W_gate, W_up, W_down, dy):
    """Gradients of <dy, FFN(x)> for FFN(x) = W_down (SiLU(W_gate x) * (W_up x)),
    rows of x (and of dy) are tokens.

      a = x W_gate^T, b = x W_up^T, h = SiLU(a) * b, y = h W_down^T
      dh = dy W_down                  (Dgrad of the down projection)
      dW_down = dy^T h                (Wgrad of the down projection)
      da = dh * b * SiLU'(a),  db = dh * SiLU(a)
      dx = da W_gate + db W_up        (Dgrad of the gate/up projection)
      dW_gate = da^T x, dW_up = db^T x  (Wgrad of the gate/up projection)

    Returns (dx [R,d], dW_gate [I,d], dW_up [I,d], dW_down [d,I], da, db)."""
    x = np.asarray(x, np.float64)
    Wg = np.asarray(W_gate, np.float64)
    Wu = np.asarray(W_up, np.float64)
    Wd = np.asarray(W_down, np.float64)
    dy = np.asarray(dy, np.float64)
    a = x @ Wg.T
    b = x @ Wu.T
    h = silu(a) * b
    dh = dy @ Wd
    dW_down = dy.T @ h
    da = dh * b * silu_grad(a)
    db = dh * silu(a)
    dx = da @ Wg + db @ Wu
    return dx, da.T @ x, db.T @ x, dW_down, da, db


def gate_backward(s_sel, d_gate):
    """g_k = s_k / S with S = sum_j s_j over the selected experts (reading R1):
    dL/ds_j = sum_k dL/dg_k * (delta_jk / S - s_k / S^2)
            = (dL/dg_j - sum_k g_k dL/dg_k) / S."""
    s_sel = np.asarray(s_sel, np.float64)
    d_gate = np.asarray(d_gate, np.float64)
    S = s_sel.sum(axis=1, keepdims=True)
    g = s_sel / S
    return (d_gate - (g * d_gate).sum(axis=1, keepdims=True)) / S


def layer_backward(u, E, idx, routed, shared, dh):
    """Backward of h'_t = u_t + sum_s FFN_s(u_t) + sum_{i in S_t} g_{i,t} FFN_i(u_t),
    g from s_{i,t} = Sigmoid(u_t^T e_i) over the fixed selection idx (B1).

    routed[e] / shared[j] yield (W_gate, W_up, W_down).  Returns a dict:
      du [T,d], dE [N_r,d], d_gate [T,K] (dL/dg), d_logit [T,K] (dL/d(u^T e)),
      routed: {e: (dW_gate, dW_up, dW_down)} for every expert with tokens,
      shared: [(dW_gate, dW_up, dW_down)] per shared expert.
    """
    u = np.asarray(u, np.float64)
    E = np.asarray(E, np.float64)
    dh = np.asarray(dh, np.float64)
    idx = np.asarray(idx)
    T, K = idx.shape

    # router forward quantities on the selected experts (float64, B2)
    logit_sel = np.einsum("td,tkd->tk", u, E[idx])
    s_sel = sigmoid(logit_sel)
    g = s_sel / s_sel.sum(axis=1, keepdims=True)

    du = dh.copy()                                   # residual path
    out_shared = []
    for j in range(len(shared)):
        dx, dWg, dWu, dWd, _, _ = swiglu_ffn_backward(u, *shared[j], dh)
        du += dx
        out_shared.append((dWg, dWu, dWd))

    d_gate = np.zeros((T, K))
    out_routed = {}
    for e in np.unique(idx):
        t, k = np.nonzero(idx == e)                  # one slot per token for expert e
        W = routed[int(e)]
        y = swiglu_ffn(u[t], *W)
        d_gate[t, k] = np.sum(dh[t] * y, axis=1)     # dL/dg = <dh', FFN_e(u_t)>
        dx, dWg, dWu, dWd, _, _ = swiglu_ffn_backward(u[t], *W, g[t, k][:, None] * dh[t])
        du[t] += dx
        out_routed[int(e)] = (dWg, dWu, dWd)

    ds = gate_backward(s_sel, d_gate)
    d_logit = ds * s_sel * (1.0 - s_sel)             # Sigmoid' = s (1 - s)
    du += np.einsum("tk,tkd->td", d_logit, E[idx])
    dE = np.zeros_like(E)
    np.add.at(dE, idx.reshape(-1), d_logit.reshape(-1, 1) * np.repeat(u, K, axis=0))
    return {"du": du, "dE": dE, "d_gate": d_gate, "d_logit": d_logit,
            "routed": out_routed, "shared": out_shared}


# ----------------------------------------------------------------------------
# FP8 backward (reading B5)
# ----------------------------------------------------------------------------

def quant_128x1_grouped(X, offsets):
    """Wgrad operand quantisation: for each group g (rows offsets[g] ..
    offsets[g+1]) and each block of 128 consecutive rows starting at the
    group's first row, one float32 scale per column = amax/448 over the
    block's rows (1 for an all-zero column).  Returns (q [R, D] float64 E4M3
    values, scale [n_blocks, D] float32, blocks: list of (group, r0, r1))."""
    X = np.asarray(X, np.float32)
    offsets = np.asarray(offsets)
    q = np.zeros(X.shape, np.float64)
    scales, blocks = [], []
    for g in range(len(offsets) - 1):
        for r0 in range(int(offsets[g]), int(offsets[g + 1]), FP8_TILE):
            r1 = min(r0 + FP8_TILE, int(offsets[g + 1]))
            sc = tile_scale(np.abs(X[r0:r1]).max(axis=0))
            q[r0:r1] = e4m3_round((X[r0:r1] / sc[None, :]).astype(np.float32))
            scales.append(sc)
            blocks.append((g, r0, r1))
    D = X.shape[1]
    sc = np.stack(scales) if scales else np.zeros((0, D), np.float32)
    return q, sc, blocks


def fp8_wgrad(qa, sa, qb, sb, blocks, n_groups):
    """C[g][m, n] = sum over g's blocks b of
         (sum_{r in b} qa[r, m] qb[r, n]) * sa[b, m] * sb[b, n]   (float64)."""
    qa = np.asarray(qa, np.float64)
    qb = np.asarray(qb, np.float64)
    out = np.zeros((n_groups, qa.shape[1], qb.shape[1]))
    for i, (g, r0, r1) in enumerate(blocks):
        part = qa[r0:r1].T @ qb[r0:r1]
        out[g] += part * np.asarray(sa, np.float64)[i][:, None] \
                       * np.asarray(sb, np.float64)[i][None, :]
    return out


def fp8_dgrad(q_dy, s_dy, qW, sW):
    """dh[r, n] = sum_kb (sum_{k in kb} q_dy[r, k] qW[k, n]) * s_dy[r, kb] * sW[kb, n // 128]
    for a weight W stored [K, N] with its 128x128 block scales sW [K/128, N/128]:
    the promoted GEMM against the transposed weight (same blocks, transposed)."""
    return fp8_promoted_gemm(q_dy, s_dy, np.asarray(qW).T, np.asarray(sW).T)


def fp8_swiglu_ffn_backward(x, Wq, dy):
    """Backward of fp8_swiglu_ffn for one expert's rows x [R, d] (one group) and
    upstream dy [R, d], under reading B5.  Wq: quantise_expert(...) dict.
    Returns (dx [R, d], dW_gate [I, d], dW_up [I, d], dW_down [d, I])."""
    x = np.asarray(x, np.float32)
    R = x.shape[0]
    qx, sx = quant_1x128(x)
    a = fp8_promoted_gemm(qx, sx, *Wq["gate"])
    b = fp8_promoted_gemm(qx, sx, *Wq["up"])
    I = a.shape[1]
    h = (silu(a) * b).astype(np.float32)
    dy32 = np.asarray(dy, np.float32)
    q_dy, s_dy = quant_1x128(dy32)
    qWd, sWd = Wq["down"]                           # W_down [d, I]: K = d rows, N = I cols
    dh = fp8_promoted_gemm(q_dy, s_dy, qWd.T, sWd.T)
    dA = np.concatenate([dh * b * silu_grad(a), dh * silu(a)], axis=1).astype(np.float32)
    q_dA, s_dA = quant_1x128(dA)
    qWgu = np.concatenate([Wq["gate"][0], Wq["up"][0]])   # [2I, d]: K = 2I rows, N = d cols
    sWgu = np.concatenate([Wq["gate"][1], Wq["up"][1]])
    dx = fp8_promoted_gemm(q_dA, s_dA, qWgu.T, sWgu.T)
    off = np.array([0, R])
    qa, sa, blk = quant_128x1_grouped(dy32, off)
    qb, sb, _ = quant_128x1_grouped(h, off)
    dW_down = fp8_wgrad(qa, sa, qb, sb, blk, 1)[0]
    qa, sa, _ = quant_128x1_grouped(dA, off)
    qb, sb, _ = quant_128x1_grouped(x, off)
    dW_gu = fp8_wgrad(qa, sa, qb, sb, blk, 1)[0]
    return dx, dW_gu[:I], dW_gu[I:], dW_down


def layer_backward_fp8(u, E, idx, routed_q, shared_q, dh):
    """layer_backward with every expert FFN (forward output for dL/dg, and
    its backward) evaluated under the FP8 recipe; residual, gates and router
    in float64.  routed_q[e] / shared_q[j]: quantise_expert(...) dicts.
    Returns du, dE, d_gate, d_logit and the routed / shared weight gradients."""
    u = np.asarray(u, np.float64)
    E = np.asarray(E, np.float64)
    dh = np.asarray(dh, np.float64)
    idx = np.asarray(idx)
    T, K = idx.shape
    logit_sel = np.einsum("td,tkd->tk", u, E[idx])
    s_sel = sigmoid(logit_sel)
    g = s_sel / s_sel.sum(axis=1, keepdims=True)
    du = dh.copy()
    out_shared = []
    for j in range(len(shared_q)):
        dx, dWg, dWu, dWd = fp8_swiglu_ffn_backward(u, shared_q[j], dh)
        du += dx
        out_shared.append((dWg, dWu, dWd))
    d_gate = np.zeros((T, K))
    out_routed = {}
    for e in np.unique(idx):
        t, k = np.nonzero(idx == e)
        Wq = routed_q[int(e)]
        y = fp8_swiglu_ffn(u[t], Wq)
        d_gate[t, k] = np.sum(dh[t] * y, axis=1)
        dx, dWg, dWu, dWd = fp8_swiglu_ffn_backward(u[t], Wq, g[t, k][:, None] * dh[t])
        du[t] += dx
        out_routed[int(e)] = (dWg, dWu, dWd)
    ds = gate_backward(s_sel, d_gate)
    d_logit = ds * s_sel * (1.0 - s_sel)
    du += np.einsum("tk,tkd->td", d_logit, E[idx])
    dE = np.zeros_like(E)
    np.add.at(dE, idx.reshape(-1), d_logit.reshape(-1, 1) * np.repeat(u, K, axis=0))
    return {"du": du, "dE": dE, "d_gate": d_gate, "d_logit": d_logit,
            "routed": out_routed, "shared": out_shared}
