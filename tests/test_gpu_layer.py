"""Whole-layer parity on the five synthetic configurations: the GPU layer
(route -> permute -> routed and shared FFNs -> combine -> bias update, all
through the C ABI) against the CPU oracle.  Routing is compared for every
token; h' in full for the small shapes and on a seeded token sample for the
V3 shapes, in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_60_b200.configs import CONFIGS
from mixture_experts_layer_60_b200.layer import MoELayer
from mixture_experts_layer_60_b200.synth import make_layer_inputs, step_u
from oracle import moe_oracle as O
from tests.harness import (GATE_TOL, TOL, LazyExperts, assert_close, check_routing,
                           check_whole_experts, f64, grouped_reference, oracle_layer_rows)

pytestmark = pytest.mark.gpu


def _oracle_layer(cfg, w, u_rows, idx, gate):
    routed = LazyExperts(w["W_gate_up"], w["W_down"])
    shared = LazyExperts(w["Ws_gate_up"], w["Ws_down"])
    if cfg.dtype == "e4m3":
        rq = _QuantExperts(routed)
        sq = _QuantExperts(shared)
        return O.layer_forward_fp8(u_rows, idx, gate, rq, sq)
    return O.layer_forward(u_rows, idx, gate, routed, shared)


class _QuantExperts:
    def __init__(self, ex):
        self.ex = ex

    def __len__(self):
        return len(self.ex)

    def __getitem__(self, e):
        g, u, d = self.ex[e]
        return O.quantise_expert(g.astype(np.float32), u.astype(np.float32), d.astype(np.float32))


def _run(cfg, T=None, sample=None, seed_sample=0):
    w = make_layer_inputs(cfg, "cuda", T=T)
    u = w["u"]
    layer = MoELayer(cfg, w, T_max=u.shape[0])
    h = layer.forward(u)
    torch.cuda.synchronize()
    if cfg.n_groups > 1:
        ref = O.route_grouped(f64(u), f64(w["E"]), w["b"].cpu().numpy(), cfg.K, cfg.n_groups,
                              cfg.topk_groups)
        ref_chk = grouped_reference(ref, cfg.K, cfg.n_groups, cfg.topk_groups)
    else:
        ref = ref_chk = O.route(f64(u), f64(w["E"]), w["b"].cpu().numpy(), cfg.K)
    exempt, idx, gate = check_routing(layer.topk_idx.cpu().numpy(), layer.topk_gate.cpu().numpy(),
                                      layer.counts.cpu().numpy(), ref_chk, cfg.K,
                                      gate_tol=GATE_TOL[cfg.dtype])
    if cfg.n_groups > 1:
        gsz = cfg.N_r // cfg.n_groups
        used = [len(set((r // gsz).tolist())) for r in layer.topk_idx.cpu().numpy()]
        assert max(used) <= cfg.topk_groups
    Tn = u.shape[0]
    rows = np.arange(Tn) if sample is None else \
        np.sort(np.random.default_rng(seed_sample).choice(Tn, sample, replace=False))
    if sample is None:
        want = _oracle_layer(cfg, w, f64(u)[rows], idx[rows], gate[rows])
    else:
        want = oracle_layer_rows(w, rows, idx[rows], gate[rows], fp8=cfg.dtype == "e4m3")
    got = f64(h)[rows]
    err = assert_close(got, want, TOL[cfg.dtype], f"h' {cfg.name}")
    return layer, w, err, exempt


def _three_experts(layer):
    """The most-loaded expert, the least-loaded non-empty one and a median one."""
    c = layer.counts.cpu().numpy()
    nz = np.nonzero(c)[0]
    order = nz[np.argsort(c[nz], kind="stable")]
    return [int(order[-1]), int(order[0]), int(order[len(order) // 2])]


def test_layer_tiny_f32():
    _run(CONFIGS["tiny_f32"])


def test_layer_small_bf16():
    _run(CONFIGS["small_bf16"])


def test_layer_v3_bf16_sampled():
    """V3 shape (T = 8192): h' on 1024 sampled tokens and every routed row of
    three whole experts (the most loaded spans several 16-row token tiles)."""
    layer, w, _, _ = _run(CONFIGS["v3_bf16"], sample=1024)
    check_whole_experts(layer, w, _three_experts(layer), TOL["bf16"])


def test_layer_v3_bf16_ragged_T():
    """T not a multiple of the 128-row tile, V3 shape."""
    _run(CONFIGS["v3_bf16"], T=1000, sample=24, seed_sample=1)


def test_layer_v3_fp8_sampled():
    """FP8 V3 shape (T = 16384, 0.1 % outliers x50) against the FP8-emulating
    oracle: h' on 1024 sampled tokens and every routed row of three whole
    experts (the most loaded spans several 128-token tiles)."""
    layer, w, _, _ = _run(CONFIGS["v3_fp8"], sample=1024, seed_sample=2)
    check_whole_experts(layer, w, _three_experts(layer), TOL["e4m3"], fp8=True)


def test_layer_v3_fp8_ragged_T():
    """FP8 at V3 width with T not a multiple of the 128-row tile (1000 tokens):
    routing of every token, h' on 64 sampled tokens."""
    _run(CONFIGS["v3_fp8"], T=1000, sample=64, seed_sample=5)


def test_layer_v3_fp8_decode_batch():
    """FP8 at V3 width with a decode-sized batch (256 tokens, ~8 per expert,
    so every 128-row expert tile is mostly padding): every token's h'."""
    _run(CONFIGS["v3_fp8"], T=256, sample=256, seed_sample=6)


def test_layer_fp8_small_full():
    """FP8 layer on a small shape, every token compared."""
    from dataclasses import replace
    cfg = replace(CONFIGS["v3_fp8"], name="fp8_small", T=1024, d=512, N_r=32, K=4, N_s=1, I=256)
    _run(cfg)


def test_layer_v3_decode_sampled():
    """Decode-shaped batch (T = 256, ~8 tokens per expert; 16-row token
    tiles): every token's h' against the oracle."""
    _run(CONFIGS["v3_decode_bf16"], sample=256, seed_sample=3)


def test_layer_v3_grouped_sampled():
    """Node-limited routing at V3 shape (8 groups of 32 experts, at most 4 per
    token): routing of every token, h' on 256 sampled tokens."""
    _run(CONFIGS["v3_grouped_bf16"], sample=256, seed_sample=4)


def test_layer_all_tokens_one_expert():
    """K = 1 and a dominant bias: one group holds every token, the others are empty."""
    cfg = CONFIGS["small_bf16"]
    w = make_layer_inputs(cfg, "cuda", T=600)
    w["b"] = torch.zeros_like(w["b"])
    w["b"][5] = 10.0
    from dataclasses import replace
    cfg1 = replace(cfg, K=1)
    layer = MoELayer(cfg1, w)
    h = layer.forward(w["u"])
    torch.cuda.synchronize()
    assert (layer.topk_idx.cpu() == 5).all()
    assert (layer.topk_gate.cpu() == 1.0).all()
    assert layer.offsets.cpu().tolist() == [0] * 6 + [600] * 59
    idx = np.full((600, 1), 5, np.int32)
    gate = np.ones((600, 1), np.float32)
    want = _oracle_layer(cfg1, w, f64(w["u"]), idx, gate)
    assert_close(f64(h), want, TOL["bf16"], "h'")


def test_bias_update_steps_and_resume():
    """Steps of forward + bias update: b follows the oracle's rule bit for bit
    from the GPU's load, and a run split in two with b saved and reloaded in
    between equals the uninterrupted run."""
    cfg = CONFIGS["small_bf16"]
    from dataclasses import replace
    cfg = replace(cfg, T=512)
    w = make_layer_inputs(cfg, "cuda", T=512)
    a = MoELayer(cfg, w)
    b_hist = []
    for s in range(6):
        u = step_u(cfg, s, "cuda", T=512)
        b_before = a.b.cpu().numpy().copy()
        a.step(u)
        torch.cuda.synchronize()
        want = O.bias_update(b_before, a.counts.cpu().numpy(), 512, cfg.K)
        np.testing.assert_array_equal(a.b.cpu().numpy(), want)
        b_hist.append(a.b.clone())
    # resume: 3 steps, save b, fresh layer, 3 more
    b1 = MoELayer(cfg, w)
    for s in range(3):
        b1.step(step_u(cfg, s, "cuda", T=512))
    saved = b1.b.cpu().clone()
    w2 = dict(w)
    w2["b"] = saved.to("cuda")
    b2 = MoELayer(cfg, w2)
    for s in range(3, 6):
        h2 = b2.step(step_u(cfg, s, "cuda", T=512))
    torch.cuda.synchronize()
    assert torch.equal(b2.b, b_hist[-1])
    a_last = MoELayer(cfg, dict(w, b=b_hist[-2]))
    h_re = a_last.forward(step_u(cfg, 5, "cuda", T=512))
    torch.cuda.synchronize()
    assert torch.equal(h2, h_re)


def test_skewed_load_steps_route_and_balance():
    """Skewed-popularity V3 shape: each step's routing equals the oracle's
    (with the bias the GPU carries), the bias follows the oracle's rule bit for
    bit from the GPU's load, the load is skewed at the start, and a run of
    4 + 4 steps with the bias saved and reloaded equals 8 steps bit for bit."""
    from dataclasses import replace
    cfg = replace(CONFIGS["v3_zipf_bf16"], T=1024)
    w = make_layer_inputs(cfg, "cuda")
    a = MoELayer(cfg, w)
    E = f64(w["E"])
    first_ratio = None
    for s in range(8):
        u = step_u(cfg, s, "cuda")
        b_before = a.b.cpu().numpy().copy()
        a.step(u)
        torch.cuda.synchronize()
        ref = O.route(f64(u), E, b_before, cfg.K)
        check_routing(a.topk_idx.cpu().numpy(), a.topk_gate.cpu().numpy(),
                      a.counts.cpu().numpy(), ref, cfg.K, gate_tol=GATE_TOL["bf16"])
        np.testing.assert_array_equal(a.b.cpu().numpy(),
                                      O.bias_update(b_before, a.counts.cpu().numpy(), cfg.T, cfg.K))
        if s == 0:
            first_ratio = a.counts.max().item() / (cfg.T * cfg.K / cfg.N_r)
    assert first_ratio > 4.0, first_ratio          # the recipe does skew the load
    b_half = MoELayer(cfg, w)
    for s in range(4):
        b_half.step(step_u(cfg, s, "cuda"))
    w2 = dict(w, b=b_half.b.clone())
    b2 = MoELayer(cfg, w2)
    for s in range(4, 8):
        b2.step(step_u(cfg, s, "cuda"))
    torch.cuda.synchronize()
    assert torch.equal(b2.b, a.b)


def test_host_stepper_overlapped_equals_device_steps():
    """Steps fed from pinned host memory with uploads and downloads overlapped
    on copy streams give, step for step, the same h' (bit for bit) and the same
    final bias as the same steps run on device-resident tokens."""
    from dataclasses import replace
    from mixture_experts_layer_60_b200.hostio import HostStepper
    cfg = replace(CONFIGS["small_bf16"], T=768)
    w = make_layer_inputs(cfg, "cuda", T=768)
    n = 5
    us = [step_u(cfg, s, "cuda", T=768) for s in range(n)]
    ref = MoELayer(cfg, w)
    want = []
    for u in us:
        want.append(ref.step(u).cpu().clone())
    lay = MoELayer(cfg, w)
    st = HostStepper(cfg.T, cfg.d, us[0].dtype, "cuda")
    u_h = [u.cpu().pin_memory() for u in us]
    h_h = [torch.empty_like(x).pin_memory() for x in u_h]

    def fn(u_in, out):
        lay.forward(u_in, out=out)
        lay.bias_update()

    st.run(u_h, h_h, fn)
    torch.cuda.synchronize()
    for s in range(n):
        assert torch.equal(h_h[s], want[s]), s
    assert torch.equal(lay.b, ref.b)


def test_skewed_load_full_shape_routing_and_bias():
    """The skewed-popularity V3 configuration at its full shape (T = 8192,
    Zipf(1.2) centroid norms): for 3 steps of forward + bias update with fresh
    tokens, every token's routing equals the oracle's (with the bias the GPU
    carries) bit for bit except genuine near-ties (key gap < 1e-6), the load
    matches, b follows the oracle's rule bit for bit, and every routed row of
    the most-loaded expert (thousands of rows, many token tiles) and two more
    matches the oracle's FFN."""
    cfg = CONFIGS["v3_zipf_bf16"]
    w = make_layer_inputs(cfg, "cuda")
    a = MoELayer(cfg, w)
    E = f64(w["E"])
    for s in range(3):
        u = step_u(cfg, s, "cuda")
        b_before = a.b.cpu().numpy().copy()
        a.step(u)
        torch.cuda.synchronize()
        ref = O.route(f64(u), E, b_before, cfg.K)
        check_routing(a.topk_idx.cpu().numpy(), a.topk_gate.cpu().numpy(),
                      a.counts.cpu().numpy(), ref, cfg.K, gate_tol=GATE_TOL["bf16"])
        np.testing.assert_array_equal(a.b.cpu().numpy(),
                                      O.bias_update(b_before, a.counts.cpu().numpy(), cfg.T, cfg.K))
    assert a.counts.max().item() > 4 * cfg.T * cfg.K / cfg.N_r       # the load is skewed
    w_step = dict(w, u=u)
    check_whole_experts(a, w_step, _three_experts(a), TOL["bf16"])


def test_skewed_load_full_protocol_100_steps():
    """The skewed-popularity configuration's whole protocol: T = 8192 fresh
    tokens per step for 100 steps of forward + bias update.  At every step
    each token's routing equals the oracle's with the bias the GPU carries
    (bit for bit except genuine near-ties), the load matches, and b follows
    the oracle's rule bit for bit; over the run the bias lowers the
    max/mean expert load."""
    cfg = CONFIGS["v3_zipf_bf16"]
    w = make_layer_inputs(cfg, "cuda")
    a = MoELayer(cfg, w)
    E = f64(w["E"])
    mean = cfg.T * cfg.K / cfg.N_r
    ratios = []
    for s in range(100):
        u = step_u(cfg, s, "cuda")
        b_before = a.b.cpu().numpy().copy()
        a.step(u)
        torch.cuda.synchronize()
        counts = a.counts.cpu().numpy()
        ref = O.route(f64(u), E, b_before, cfg.K)
        check_routing(a.topk_idx.cpu().numpy(), a.topk_gate.cpu().numpy(), counts, ref, cfg.K,
                      gate_tol=GATE_TOL["bf16"])
        np.testing.assert_array_equal(a.b.cpu().numpy(),
                                      O.bias_update(b_before, counts, cfg.T, cfg.K))
        ratios.append(counts.max() / mean)
    assert ratios[0] > 4.0, ratios[0]
    assert np.mean(ratios[-10:]) < np.mean(ratios[:10]), (ratios[:10], ratios[-10:])
