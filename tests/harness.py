"""Shared helpers of the parity tests: host copies of device tensors for the
oracle, routing comparison with the near-tie exemption, tolerance checks."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O

# Output tolerances, as fractions of max|reference| (float32, bfloat16, FP8 recipe).
TOL = {"f32": 1e-5, "bf16": 2e-2, "e4m3": 6e-2}
TIE_GAP = 1e-6   # routing may legitimately differ where two keys are closer than this
# Gate tolerance (fraction of max|gate|).  float32 inputs: the GPU's logits
# differ from the oracle's only by float32 rounding.  bf16 inputs: the logits
# are float32 sums of d bf16 x bf16 products (tensor cores); at d = 7168 with
# centroid norms up to 5 (the skewed recipe) a logit of magnitude ~15 carries
# an absolute error up to ~1e-4, so s = Sigmoid(x) moves by up to ~2.5e-5 and
# g = s / sum(s) by about the same: 1e-4 of max|g| covers it.
GATE_TOL = {"f32": 1e-5, "bf16": 1e-4, "e4m3": 1e-4}


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a device tensor (bf16/f32 values are representable)."""
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, ref, tol, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max() if got.size else 0.0
    assert err <= tol * scale + 1e-30, f"{what}: max|err| {err:.3e} > {tol} * max|ref| {scale:.3e}"
    return err / max(scale, 1e-30)


class LazyExperts:
    """Expert weights for the oracle, copied from the device one expert at a
    time: item e -> (W_gate [I,d], W_up [I,d], W_down [d,I]) as float64."""

    def __init__(self, W_gate_up: torch.Tensor, W_down: torch.Tensor):
        self.gu, self.dn = W_gate_up, W_down
        self.I = W_gate_up.shape[1] // 2

    def __len__(self):
        return self.gu.shape[0]

    def __getitem__(self, e):
        gu = f64(self.gu[e])
        return gu[:self.I], gu[self.I:], f64(self.dn[e])


def check_routing(idx_gpu, gate_gpu, counts_gpu, ref, K, gate_tol=TOL["f32"]):
    """Routing must equal the oracle's except on near-tie tokens.

    Returns (mask of tokens whose selection is exempt, merged idx, merged gate):
    the merged routing is the oracle's, except that exempt tokens take the
    GPU's selection after it is checked to be a valid top-K within TIE_GAP."""
    idx_gpu = np.asarray(idx_gpu)
    gate_gpu = np.asarray(gate_gpu)
    key = ref["key"]
    sel_gap, ord_gap = O.topk_margins(key, ref["idx"])
    sel_tie = sel_gap < TIE_GAP
    ord_tie = ord_gap < TIE_GAP
    exact = ~(sel_tie | ord_tie)
    assert np.array_equal(idx_gpu[exact], ref["idx"][exact]), \
        f"{int((idx_gpu[exact] != ref['idx'][exact]).any(1).sum())} tokens routed differently"
    only_order = ord_tie & ~sel_tie
    assert np.array_equal(np.sort(idx_gpu[only_order], 1), np.sort(ref["idx"][only_order], 1))
    # exempt tokens: the GPU's K experts must be a top-K of the keys up to TIE_GAP
    for t in np.nonzero(sel_tie)[0]:
        ks = key[t]
        kth = np.sort(ks)[::-1][K - 1]
        assert len(set(idx_gpu[t].tolist())) == K
        assert np.all(ks[idx_gpu[t]] >= kth - TIE_GAP)
    # load: exact where no selection tie, else consistent with the GPU's own routing
    counts_gpu = np.asarray(counts_gpu)
    assert np.array_equal(counts_gpu, np.bincount(idx_gpu.reshape(-1), minlength=len(counts_gpu)))
    if not sel_tie.any():
        assert np.array_equal(counts_gpu, ref["counts"])
    same = np.all(idx_gpu == ref["idx"], axis=1)
    if same.any():
        assert_close(gate_gpu[same], ref["gate"][same], gate_tol, "gates")
    merged_idx = ref["idx"].copy()
    merged_idx[sel_tie | ord_tie] = idx_gpu[sel_tie | ord_tie]
    merged_gate = ref["gate"].copy()
    merged_gate[sel_tie | ord_tie] = O.gates(ref["s"], idx_gpu)[sel_tie | ord_tie]
    return sel_tie | ord_tie, merged_idx, merged_gate


def grouped_reference(ref, K, n_groups, topk_groups):
    """Reference routing reshaped so that check_routing exempts grouped near-ties:
    keys outside the oracle's kept groups become -inf, and tokens whose
    topk_groups-th and next group scores are closer than TIE_GAP get a zero
    margin (their kept groups may legitimately differ)."""
    key = ref["key"]
    T, N_r = key.shape
    gs = N_r // n_groups
    g = key.reshape(T, n_groups, gs).max(axis=2)
    gsrt = -np.sort(-g, axis=1)
    gtie = (gsrt[:, topk_groups - 1] - gsrt[:, topk_groups]) < TIE_GAP if topk_groups < n_groups \
        else np.zeros(T, bool)
    kept = np.zeros((T, n_groups), bool)
    np.put_along_axis(kept, np.argsort(-g, axis=1, kind="stable")[:, :topk_groups], True, axis=1)
    masked = np.where(np.repeat(kept, gs, axis=1), key, -np.inf).astype(np.float32)
    # group-score near-tie: give the excluded experts the K-th key, so the gap
    # between the K-th and (K+1)-th key is zero and the token is exempt
    if gtie.any():
        kth = -np.sort(-masked[gtie], axis=1)[:, K - 1:K]
        masked[gtie] = np.where(np.isinf(masked[gtie]), kth, masked[gtie])
    out = dict(ref)
    out["key"] = masked
    return out


def oracle_layer_rows(w, rows, idx, gate, fp8=False):
    """h' of the tokens `rows` of w["u"] (routing idx, gate for those rows) by
    the C++ oracle, one expert at a time: each selected or shared expert's
    stored weights are copied to the host only while it is evaluated.
    float64 [len(rows), d]."""
    from oracle import moe_ref as R
    dev = w["u"].device
    u = w["u"][torch.as_tensor(np.asarray(rows), device=dev)].cpu()
    out = f64(u)
    for j in range(w["Ws_gate_up"].shape[0]):
        out += R.expert_ffn(u, w["Ws_gate_up"][j].cpu(), w["Ws_down"][j].cpu(), fp8=fp8)
    idx = np.asarray(idx)
    gate = np.asarray(gate, np.float64)
    for e in np.unique(idx):
        t, k = np.nonzero(idx == e)
        y = R.expert_ffn(u[torch.from_numpy(t)], w["W_gate_up"][int(e)].cpu(),
                         w["W_down"][int(e)].cpu(), fp8=fp8)
        out[t] += gate[t, k][:, None] * y
    return out


def check_whole_experts(layer, w, experts, tol, fp8=False):
    """Every grouped row of each expert in `experts` (the routed FFN output
    y_perm of the last forward) against the C++ oracle's FFN of the same
    token rows, within tol of max|ref| per expert."""
    from oracle import moe_ref as R
    off = layer.offsets.cpu().numpy()
    src = layer.perm_src.cpu().numpy()
    errs = {}
    for e in experts:
        a, b = int(off[e]), int(off[e + 1])
        if b == a:
            continue
        u = w["u"][torch.from_numpy(src[a:b]).to(w["u"].device)].cpu()
        want = R.expert_ffn(u, w["W_gate_up"][e].cpu(), w["W_down"][e].cpu(), fp8=fp8)
        errs[int(e)] = assert_close(f64(layer.y_perm[a:b]), want, tol, f"expert {e} rows")
    return errs
