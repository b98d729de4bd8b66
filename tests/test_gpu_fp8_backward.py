"""FP8 backward parity (reading B5 of the backward oracle): the group-aligned
128x1 Wgrad quantiser bit for bit, the FP8 Dgrad/Wgrad grouped GEMMs and the
FP8 layer backward against the FP8-emulating float64 oracle."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_60_b200 import moe_quantize_128x1_grouped
from oracle import moe_backward as B
from tests.harness import f64

pytestmark = pytest.mark.gpu


def _e4m3(q):
    return q.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("sizes", [[0, 3, 128, 130, 0, 257, 64], [1000]])
def test_quantize_128x1_grouped_bit_exact(sizes):
    rows, cols = int(sum(sizes)), 384
    g = torch.Generator(device="cuda")
    g.manual_seed(31)
    x = (torch.randn(rows, cols, generator=g, device="cuda") *
         torch.rand(1, cols, generator=g, device="cuda") * 10).to(torch.bfloat16)
    x[:, 7] = 0                                         # all-zero column: scale 1
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    nb_cap = (rows + 127) // 128 + len(sizes)
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    sc = torch.full((nb_cap, cols), -1.0, device="cuda")
    bs = torch.empty(len(sizes) + 1, dtype=torch.int32, device="cuda")
    moe_quantize_128x1_grouped(x, off, q, sc, bs)
    torch.cuda.synchronize()
    qo, so, blocks = B.quant_128x1_grouped(f64(x).astype(np.float32), off.cpu().numpy())
    nb = len(blocks)
    assert int(bs[-1]) == nb
    want_start, k = [], 0
    for gi in range(len(sizes)):
        want_start.append(k)
        k += (sizes[gi] + 127) // 128
    np.testing.assert_array_equal(bs.cpu().numpy()[:-1], want_start)
    np.testing.assert_array_equal(sc[:nb].cpu().numpy(), so)
    np.testing.assert_array_equal(_e4m3(q), qo)


# FP8 backward tolerance: GPU and oracle quantise the same recipe but from
# inputs that differ by float32/bf16 rounding (dA from float32 TMEM sums and
# bf16 pre-activations), so a few elements land one E4M3 step (2^-3 relative
# at most) apart; the bound is on max|err| / max|ref| and on the rms error.
FP8_BWD_MAX = 0.1
FP8_BWD_RMS = 0.03


def _close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), what
    scale = np.abs(ref).max()
    mx = np.abs(got - ref).max() / scale
    rms = np.sqrt(np.mean((got - ref) ** 2) / np.mean(ref ** 2))
    assert mx <= FP8_BWD_MAX and rms <= FP8_BWD_RMS, f"{what}: max {mx:.3e} rms {rms:.3e}"
    return mx, rms


@pytest.mark.parametrize("sizes", [[0, 1, 15, 127, 128, 129, 300, 40], [640]])
def test_fp8_expert_ffn_backward_ragged_groups(sizes):
    from mixture_experts_layer_60_b200 import (MOE_E4M3, moe_expert_ffn_backward,
                                               moe_expert_ffn_backward_workspace_size,
                                               moe_expert_gate_up_save, moe_quantize_128x128,
                                               moe_quantize_1x128)
    from oracle import moe_oracle as O
    d, I = 512, 256
    G, rows = len(sizes), int(sum(sizes))
    g = torch.Generator(device="cuda")
    g.manual_seed(41)
    rn = lambda *s, std=1.0: (torch.randn(*s, generator=g, device="cuda") * std).to(torch.bfloat16)
    x, dy = rn(rows, d), rn(rows, d, std=0.05)
    Wgu, Wdn = rn(G, 2 * I, d, std=d ** -0.5), rn(G, d, I, std=I ** -0.5)
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    q8 = lambda w: (torch.empty(w.shape, dtype=torch.uint8, device="cuda"),
                    torch.empty(w.shape[0], w.shape[1] // 128, w.shape[2] // 128, device="cuda"))
    (Wgu_q, sgu), (Wdn_q, sdn) = q8(Wgu), q8(Wdn)
    moe_quantize_128x128(Wgu, Wgu_q, sgu)
    moe_quantize_128x128(Wdn, Wdn_q, sdn)
    x_q = torch.empty(rows, d, dtype=torch.uint8, device="cuda")
    x_s = torch.empty(rows, d // 128, device="cuda")
    moe_quantize_1x128(x, x_q, x_s)
    h = torch.empty(rows, I, dtype=torch.uint8, device="cuda")
    h_s = torch.empty(rows, I // 128, device="cuda")
    a_gu = torch.empty(rows, 2 * I, dtype=torch.bfloat16, device="cuda")
    moe_expert_gate_up_save(x_q, off, Wgu_q, h, a_gu, x_scale=x_s, w_scale_gate_up=sgu,
                            h_scale=h_s)
    dx = torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dWgu = torch.full(Wgu.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    dWdn = torch.full(Wdn.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe_expert_ffn_backward_workspace_size(MOE_E4M3, rows, d, I, G),
                     dtype=torch.uint8, device="cuda")
    moe_expert_ffn_backward(x, off, Wgu_q, Wdn_q, a_gu, None, dy, dx, dWgu, dWdn, ws,
                            w_scale_gate_up=sgu, w_scale_down=sdn)
    torch.cuda.synchronize()
    o = off.cpu().numpy()
    for e in range(G):
        r0, r1 = o[e], o[e + 1]
        if r1 == r0:
            assert not dWgu[e].any() and not dWdn[e].any()
            continue
        Q = O.quantise_expert(f64(Wgu[e][:I]).astype(np.float32), f64(Wgu[e][I:]).astype(np.float32),
                              f64(Wdn[e]).astype(np.float32))
        dxe, dWg, dWu, dWd = B.fp8_swiglu_ffn_backward(f64(x[r0:r1]).astype(np.float32), Q,
                                                       f64(dy[r0:r1]).astype(np.float32))
        _close(f64(dx[r0:r1]), dxe, f"dx group {e}")
        _close(f64(dWgu[e][:I]), dWg, f"dW_gate group {e}")
        _close(f64(dWgu[e][I:]), dWu, f"dW_up group {e}")
        _close(f64(dWdn[e]), dWd, f"dW_down group {e}")


def test_fp8_layer_backward_small():
    from mixture_experts_layer_60_b200.configs import LayerConfig
    from mixture_experts_layer_60_b200.layer import MoELayer
    from mixture_experts_layer_60_b200.synth import make_layer_inputs, upstream_grad
    from oracle import moe_oracle as O
    from tests.harness import LazyExperts
    cfg = LayerConfig("bwd_fp8_small", T=384, d=512, N_r=8, K=2, N_s=1, I=256, dtype="e4m3",
                      seed=23, outlier_frac=0.001, outlier_scale=50.0)
    w = make_layer_inputs(cfg, "cuda")
    lay = MoELayer(cfg, w)
    h = lay.forward_train(w["u"])
    h_plain = MoELayer(cfg, w).forward(w["u"])
    dh = upstream_grad(cfg, "cuda")
    lay.backward(dh)
    torch.cuda.synchronize()
    assert torch.equal(h, h_plain), "forward_train must give the forward's h'"

    class _Q:
        def __init__(self, ex):
            self.ex = ex

        def __len__(self):
            return len(self.ex)

        def __getitem__(self, e):
            a, b, c = self.ex[e]
            return O.quantise_expert(a.astype(np.float32), b.astype(np.float32),
                                     c.astype(np.float32))

    ref = B.layer_backward_fp8(f64(w["u"]), f64(w["E"]), lay.topk_idx.cpu().numpy(),
                               _Q(LazyExperts(w["W_gate_up"], w["W_down"])),
                               _Q(LazyExperts(w["Ws_gate_up"], w["Ws_down"])), f64(dh))
    _close(f64(lay.du), ref["du"], "du")
    _close(lay.grad["E"].double().cpu().numpy(), ref["dE"], "dE")
    _close(lay.d_gate.cpu().numpy(), ref["d_gate"], "d_gate")
    I = cfg.I
    for e, (dWg, dWu, dWd) in ref["routed"].items():
        _close(f64(lay.grad["W_gate_up"][e][:I]), dWg, f"dW_gate {e}")
        _close(f64(lay.grad["W_gate_up"][e][I:]), dWu, f"dW_up {e}")
        _close(f64(lay.grad["W_down"][e]), dWd, f"dW_down {e}")
    dWg, dWu, dWd = ref["shared"][0]
    _close(f64(lay.grad["Ws_gate_up"][0][:I]), dWg, "shared dW_gate")
    _close(f64(lay.grad["Ws_down"][0]), dWd, "shared dW_down")
