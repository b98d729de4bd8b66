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

Readings (listed again in the design doc):

  B1  The selection S_t (top-K of s+b) is piecewise constant in u, E and b:
      it is held fixed and has no gradient; b receives none.  Gradient flows
      into s only through the gate values g = s_sel / sum(s_sel).
  B2  The backward is the derivative of the exact (float64) forward: s is not
      rounded to float32 here.
  B3  L = <dh, h'>: du collects the residual, the shared and routed expert
      paths and the router path.

Everything is float64.  Nothing is fused or reordered beyond the definitions.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import silu, swiglu_ffn


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
