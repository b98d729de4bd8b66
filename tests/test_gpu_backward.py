"""Backward parity: the GPU layer backward (combine backward, grouped FFN
Dgrad/Wgrad on tcgen05, unpermute, centroid gradient; all through the C ABI)
against the float64 backward oracle, on the same seeded inputs.

Kernel level: the grouped SwiGLU FFN backward on ragged groups (an empty
group, groups of 1, 15, 63, 64, 65 ... rows, so every K tail of the weight
gradient and every token tail of the Dgrad tiles is hit).  Layer level: every
gradient of a small layer in full, and the V3 shape on sampled outputs in the
launch configuration the benchmark times."""
import numpy as np
import pytest
import torch
from dataclasses import replace

from mixture_experts_layer_60_b200 import (moe_expert_ffn_backward,
                                           moe_expert_ffn_backward_workspace_size,
                                           moe_expert_gate_up, moe_expert_gate_up_save,
                                           MOE_BF16)
from mixture_experts_layer_60_b200.configs import CONFIGS, LayerConfig
from mixture_experts_layer_60_b200.layer import MoELayer
from mixture_experts_layer_60_b200.synth import make_layer_inputs, upstream_grad
from oracle import moe_backward as B
from oracle import moe_oracle as O
from tests.harness import TOL, LazyExperts, assert_close, f64

pytestmark = pytest.mark.gpu
BF = TOL["bf16"]


def _ragged_offsets(sizes):
    return torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("sizes", [[0, 1, 15, 63, 64, 65, 130, 257, 17],
                                   [700]])
def test_expert_ffn_backward_ragged_groups(sizes):
    d, I = 512, 256
    G = len(sizes)
    rows = int(sum(sizes))
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    rn = lambda *s, std=1.0: (torch.randn(*s, generator=g, device="cuda") * std).to(torch.bfloat16)
    x = rn(rows, d)
    dy = rn(rows, d, std=0.05)
    Wgu = rn(G, 2 * I, d, std=d ** -0.5)
    Wdn = rn(G, d, I, std=I ** -0.5)
    off = _ragged_offsets(sizes)
    h = torch.empty(rows, I, dtype=torch.bfloat16, device="cuda")
    h_ref = torch.empty_like(h)
    a_gu = torch.empty(rows, 2 * I, dtype=torch.bfloat16, device="cuda")
    moe_expert_gate_up_save(x, off, Wgu, h, a_gu)
    moe_expert_gate_up(x, off, Wgu, h_ref)
    dx = torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dWgu = torch.full_like(Wgu, float("nan"))
    dWdn = torch.full_like(Wdn, float("nan"))
    ws = torch.empty(moe_expert_ffn_backward_workspace_size(MOE_BF16, rows, d, I, G),
                     dtype=torch.uint8, device="cuda")
    moe_expert_ffn_backward(x, off, Wgu, Wdn, a_gu, h, dy, dx, dWgu, dWdn, ws)
    torch.cuda.synchronize()
    # the saving gate/up gives the same h as the plain one, bit for bit
    assert torch.equal(h, h_ref)
    o = off.cpu().numpy()
    xs, dys = f64(x), f64(dy)
    for e in range(G):
        r0, r1 = o[e], o[e + 1]
        Wg, Wu, Wd = f64(Wgu[e][:I]), f64(Wgu[e][I:]), f64(Wdn[e])
        if r1 == r0:
            assert not dWgu[e].any() and not dWdn[e].any(), "empty group: zero gradients"
            continue
        a_ref = xs[r0:r1] @ np.concatenate([Wg, Wu]).T
        assert_close(f64(a_gu[r0:r1]), a_ref, BF, f"pre-activations group {e}")
        dxe, dWg, dWu, dWd, _, _ = B.swiglu_ffn_backward(xs[r0:r1], Wg, Wu, Wd, dys[r0:r1])
        assert_close(f64(dx[r0:r1]), dxe, BF, f"dx group {e}")
        assert_close(f64(dWgu[e][:I]), dWg, BF, f"dW_gate group {e}")
        assert_close(f64(dWgu[e][I:]), dWu, BF, f"dW_up group {e}")
        assert_close(f64(dWdn[e]), dWd, BF, f"dW_down group {e}")


def _check_layer_backward(cfg, lay, w, dh, tokens, experts, check_shared=True):
    """Compares the GPU gradients with the oracle on `tokens` (du, d_gate,
    d_logit) and on `experts` (dW and dE rows: every token routed to them is
    included in the oracle's token set)."""
    u = w["u"]
    idx = lay.topk_idx.cpu().numpy()
    sel = set(int(t) for t in tokens)
    for e in experts:
        sel.update(np.nonzero((idx == e).any(axis=1))[0].tolist())
    S = np.array(sorted(sel))
    routed = LazyExperts(w["W_gate_up"], w["W_down"])
    shared = LazyExperts(w["Ws_gate_up"], w["Ws_down"])
    ref = B.layer_backward(f64(u)[S], f64(w["E"]), idx[S], routed, shared if check_shared else [],
                           f64(dh)[S])
    pos = {t: i for i, t in enumerate(S)}
    tk = np.array([pos[int(t)] for t in tokens])
    if check_shared:
        assert_close(f64(lay.du)[tokens], ref["du"][tk], BF, "du")
    assert_close(lay.d_gate.cpu().numpy()[tokens], ref["d_gate"][tk], BF, "d_gate")
    assert_close(lay.d_logit.cpu().numpy()[tokens], ref["d_logit"][tk], BF, "d_logit")
    I = cfg.I
    for e in experts:
        dWg, dWu, dWd = ref["routed"][e]
        assert_close(f64(lay.grad["W_gate_up"][e][:I]), dWg, BF, f"dW_gate {e}")
        assert_close(f64(lay.grad["W_gate_up"][e][I:]), dWu, BF, f"dW_up {e}")
        assert_close(f64(lay.grad["W_down"][e]), dWd, BF, f"dW_down {e}")
        assert_close(lay.grad["E"][e].double().cpu().numpy(), ref["dE"][e], BF, f"dE {e}")


def test_layer_backward_small_full():
    cfg = LayerConfig("bwd_small", T=320, d=512, N_r=16, K=4, N_s=1, I=256, dtype="bf16", seed=21,
                      bias="uniform")
    w = make_layer_inputs(cfg, "cuda")
    lay = MoELayer(cfg, w)
    h = lay.forward_train(w["u"])
    h_plain = MoELayer(cfg, w).forward(w["u"])
    dh = upstream_grad(cfg, "cuda")
    lay.backward(dh)
    torch.cuda.synchronize()
    assert torch.equal(h, h_plain), "forward_train must give the forward's h'"
    idx = lay.topk_idx.cpu().numpy()
    ref = B.layer_backward(f64(w["u"]), f64(w["E"]), idx,
                           LazyExperts(w["W_gate_up"], w["W_down"]),
                           LazyExperts(w["Ws_gate_up"], w["Ws_down"]), f64(dh))
    assert_close(f64(lay.du), ref["du"], BF, "du")
    assert_close(lay.grad["E"].double().cpu().numpy(), ref["dE"], BF, "dE")
    assert_close(lay.d_gate.cpu().numpy(), ref["d_gate"], BF, "d_gate")
    assert_close(lay.d_logit.cpu().numpy(), ref["d_logit"], BF, "d_logit")
    I = cfg.I
    for e in range(cfg.N_r):
        if e not in ref["routed"]:
            assert not lay.grad["W_gate_up"][e].any()
            continue
        dWg, dWu, dWd = ref["routed"][e]
        assert_close(f64(lay.grad["W_gate_up"][e][:I]), dWg, BF, f"dW_gate {e}")
        assert_close(f64(lay.grad["W_gate_up"][e][I:]), dWu, BF, f"dW_up {e}")
        assert_close(f64(lay.grad["W_down"][e]), dWd, BF, f"dW_down {e}")
    dWg, dWu, dWd = ref["shared"][0]
    assert_close(f64(lay.grad["Ws_gate_up"][0][:I]), dWg, BF, "shared dW_gate")
    assert_close(f64(lay.grad["Ws_gate_up"][0][I:]), dWu, BF, "shared dW_up")
    assert_close(f64(lay.grad["Ws_down"][0]), dWd, BF, "shared dW_down")


def test_layer_backward_v3_sampled():
    """V3 shape, T = 8192: du, d_gate, d_logit on 48 sampled tokens; dW and dE
    of two experts (all their tokens); the shared expert's dW_down on every
    token through sampled rows."""
    cfg = CONFIGS["v3_bf16"]
    w = make_layer_inputs(cfg, "cuda")
    lay = MoELayer(cfg, w)
    lay.forward_train(w["u"])
    dh = upstream_grad(cfg, "cuda")
    lay.backward(dh)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    tokens = np.sort(rng.choice(cfg.T, 48, replace=False))
    counts = lay.counts.cpu().numpy()
    experts = [int(np.argmax(counts)), int(np.argmin(counts))]
    _check_layer_backward(cfg, lay, w, dh, tokens, experts)
    # shared expert weight gradient over all 8192 tokens, 64 sampled rows of dW_down
    rows = np.sort(rng.choice(cfg.d, 64, replace=False))
    u, Wg, Wu = f64(w["u"]), f64(w["Ws_gate_up"][0][:cfg.I]), f64(w["Ws_gate_up"][0][cfg.I:])
    hs = O.silu(u @ Wg.T) * (u @ Wu.T)
    want = f64(dh)[:, rows].T @ hs
    assert_close(f64(lay.grad["Ws_down"][0])[rows], want, BF, "shared dW_down rows")


@pytest.mark.parametrize("N_s,K", [(0, 1), (2, 6)])
def test_layer_backward_edge_shapes(N_s, K):
    """No shared expert with K = 1, and two shared experts with K = 6; expert
    0 gets no token (bias -1), so its weight gradients must be exactly zero."""
    cfg = LayerConfig(f"bwd_edge_{N_s}_{K}", T=200, d=256, N_r=16, K=K, N_s=N_s, I=256,
                      dtype="bf16", seed=22)
    w = make_layer_inputs(cfg, "cuda")
    w["b"][0] = -1.0
    lay = MoELayer(cfg, w)
    lay.forward_train(w["u"])
    dh = upstream_grad(cfg, "cuda")
    lay.backward(dh)
    torch.cuda.synchronize()
    idx = lay.topk_idx.cpu().numpy()
    assert not (idx == 0).any()
    assert not lay.grad["W_gate_up"][0].any() and not lay.grad["W_down"][0].any()
    ref = B.layer_backward(f64(w["u"]), f64(w["E"]), idx,
                           LazyExperts(w["W_gate_up"], w["W_down"]),
                           LazyExperts(w["Ws_gate_up"], w["Ws_down"]) if N_s else [], f64(dh))
    assert_close(f64(lay.du), ref["du"], BF, "du")
    assert_close(lay.grad["E"].double().cpu().numpy(), ref["dE"], BF, "dE")
    I = cfg.I
    for e, (dWg, dWu, dWd) in ref["routed"].items():
        assert_close(f64(lay.grad["W_gate_up"][e][:I]), dWg, BF, f"dW_gate {e}")
        assert_close(f64(lay.grad["W_down"][e]), dWd, BF, f"dW_down {e}")
    for j in range(N_s):
        dWg, dWu, dWd = ref["shared"][j]
        assert_close(f64(lay.grad["Ws_gate_up"][j][I:]), dWu, BF, f"shared {j} dW_up")
        assert_close(f64(lay.grad["Ws_down"][j]), dWd, BF, f"shared {j} dW_down")
