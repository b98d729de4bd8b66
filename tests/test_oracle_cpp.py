"""The C++ oracle (oracle/moe_ref.cpp) against the hand-derived example and
against the independent numpy oracle (oracle/moe_oracle.py, itself pinned in
test_oracle_pins.py): routing, load and permutation bit for bit, the bias
update bit for bit, layer outputs (bf16, float32 and under the FP8 recipe)
within 1e-12 of max|ref| (both are float64; only summation order differs)."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import moe_ref as R

HERE = os.path.dirname(__file__)


def _sigmoid(z):
    return 1.0 / (1.0 + math.exp(-z))


def _eval(expr):
    env = {"ln": math.log, "silu": lambda z: z * _sigmoid(z), "__builtins__": {}}
    return float(eval(expr, env))  # fixture expressions only (trusted, committed file)


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _f64(t):
    return t.to(torch.float64).numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


def test_hand_example():
    """tests/golden/handworked_layer.json, derived by hand from the equations of
    section 方法 / 2: routing, gates, load, h' and the bias update."""
    with open(os.path.join(HERE, "golden", "handworked_layer.json")) as f:
        h = json.load(f)
    u = np.array(h["u"], np.float32)
    E = np.array([[_eval(x) for x in row] for row in h["E_expr"]], np.float32)
    b = np.array(h["b"], np.float32)
    r = R.route(u, E, b, h["K"])
    assert r["idx"].tolist() == h["expect"]["idx"]
    assert r["counts"].tolist() == h["expect"]["counts"]
    want_g = np.array([[_eval(x) for x in row] for row in h["expect"]["gate_expr"]])
    np.testing.assert_allclose(r["gate"], want_g, rtol=1e-6, atol=0)
    r0 = R.route(u, E, np.zeros(4, np.float32), h["K"])
    assert r0["idx"].tolist() == h["expect"]["idx_without_bias"]
    rt, st = h["routed"], h["shared"]
    routed = [(np.concatenate([np.array(rt["W_gate"][i], np.float32),
                               np.array(rt["W_up"][i], np.float32)]),
               np.array(rt["W_down"][i], np.float32)) for i in range(h["N_r"])]
    shared = [(np.concatenate([np.array(st["W_gate"][j], np.float32),
                               np.array(st["W_up"][j], np.float32)]),
               np.array(st["W_down"][j], np.float32)) for j in range(h["N_s"])]
    out = R.layer_forward(u, r["idx"], r["gate"], routed, shared)
    want_h = np.array([[_eval(x) for x in row] for row in h["expect"]["h_expr"]])
    np.testing.assert_allclose(out, want_h, rtol=1e-6, atol=1e-7)
    nb = R.bias_update(b, r["counts"], h["T"], h["K"])
    np.testing.assert_array_equal(nb, np.array([_eval(x) for x in h["expect"]["b_after_expr"]],
                                               np.float32))


@pytest.mark.parametrize("n_groups,topk_groups", [(1, 1), (4, 2), (8, 3)])
def test_route_matches_numpy_oracle(n_groups, topk_groups):
    rng = np.random.default_rng(3 + n_groups)
    T, d, N_r, K = 300, 256, 32, 6
    u = _bf16(rng.standard_normal((T, d)))
    E = _bf16(rng.standard_normal((N_r, d)) / math.sqrt(d))
    b = rng.uniform(-0.01, 0.01, N_r).astype(np.float32)
    got = R.route(u, E, b, K, n_groups, topk_groups)
    if n_groups == 1:
        want = O.route(_f64(u), _f64(E), b, K)
    else:
        want = O.route_grouped(_f64(u), _f64(E), b, K, n_groups, topk_groups)
    # s is Sigmoid of a float64 dot product rounded once to float32: the two
    # summation orders agree to float32 except at a rounding boundary
    ulp = np.spacing(want["s"])
    assert np.all(np.abs(got["s"] - want["s"]) <= ulp)
    same_s = np.all(got["s"] == want["s"], axis=1)
    assert same_s.mean() > 0.99
    np.testing.assert_array_equal(got["idx"][same_s], want["idx"][same_s])
    np.testing.assert_array_equal(got["gate"][same_s], want["gate"][same_s])
    if same_s.all():
        np.testing.assert_array_equal(got["counts"], want["counts"])


def test_permute_and_bias_match_numpy_oracle():
    rng = np.random.default_rng(8)
    T, K, N_r = 1000, 8, 64
    p = 1.0 / np.arange(1, N_r + 1) ** 1.2
    idx = np.stack([rng.choice(N_r, K, replace=False, p=p / p.sum()) for _ in range(T)])
    got = R.permute_indices(idx, N_r)
    want = O.permute_indices(idx, N_r)
    for a, b in zip(got, want):
        np.testing.assert_array_equal(a, b)
    counts = np.bincount(idx.reshape(-1), minlength=N_r).astype(np.int32)
    counts[:3] = T * K // N_r                        # equal to the mean: unchanged
    b = rng.uniform(-0.05, 0.05, N_r).astype(np.float32)
    np.testing.assert_array_equal(R.bias_update(b, counts, T, K), O.bias_update(b, counts, T, K))
    bad = idx.copy()
    bad[::9, 2] = -1
    bad[::13, 5] = N_r
    off, src, inv = R.permute_indices(bad, N_r)
    assert np.all(inv[bad < 0] == -1) and np.all(inv[bad >= N_r] == -1)
    assert off[-1] == int(((bad >= 0) & (bad < N_r)).sum())


def _experts(rng, G, d, I, conv):
    return [(conv(np.concatenate([rng.standard_normal((I, d)) / math.sqrt(d),
                                  rng.standard_normal((I, d)) / math.sqrt(d)])),
             conv(rng.standard_normal((d, I)) / math.sqrt(I))) for _ in range(G)]


def _split(w):
    gu, dn = _f64(w[0]), _f64(w[1])
    I = gu.shape[0] // 2
    return gu[:I], gu[I:], dn


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layer_matches_numpy_oracle(dtype):
    rng = np.random.default_rng(11)
    T, d, N_r, K, N_s, I = 70, 256, 12, 3, 2, 128
    conv = _bf16 if dtype == "bf16" else (lambda a: np.asarray(a, np.float32))
    u = conv(rng.standard_normal((T, d)))
    E = conv(rng.standard_normal((N_r, d)) / math.sqrt(d))
    routed, shared = _experts(rng, N_r, d, I, conv), _experts(rng, N_s, d, I, conv)
    r = R.route(u, E, np.zeros(N_r, np.float32), K)
    got = R.layer_forward(u, r["idx"], r["gate"], routed, shared)
    want = O.layer_forward(_f64(u), r["idx"], r["gate"], [_split(w) for w in routed],
                           [_split(w) for w in shared])
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()
    # an expert that no token selects may be left out
    sparse = {int(e): routed[int(e)] for e in np.unique(r["idx"])}
    np.testing.assert_array_equal(R.layer_forward(u, r["idx"], r["gate"], sparse, shared), got)


def test_fp8_layer_matches_numpy_oracle():
    rng = np.random.default_rng(12)
    T, d, N_r, K, N_s, I = 40, 256, 6, 2, 1, 256
    u = _bf16(rng.standard_normal((T, d)) * np.where(rng.random((T, d)) < 0.01, 50.0, 1.0))
    E = _bf16(rng.standard_normal((N_r, d)) / math.sqrt(d))
    routed, shared = _experts(rng, N_r, d, I, _bf16), _experts(rng, N_s, d, I, _bf16)
    r = R.route(u, E, np.zeros(N_r, np.float32), K)
    got = R.layer_forward(u, r["idx"], r["gate"], routed, shared, fp8=True)

    def q(w):
        g, up, dn = _split(w)
        return O.quantise_expert(g.astype(np.float32), up.astype(np.float32),
                                 dn.astype(np.float32))
    want = O.layer_forward_fp8(_f64(u), r["idx"], r["gate"], [q(w) for w in routed],
                               [q(w) for w in shared])
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()
    y = R.expert_ffn(u[:9], routed[0][0], routed[0][1], fp8=True)
    np.testing.assert_allclose(y, O.fp8_swiglu_ffn(_f64(u[:9]), q(routed[0])), rtol=0,
                               atol=1e-12 * np.abs(y).max())


def test_thread_count_leaves_results_unchanged():
    """The oracle's OpenMP thread count (set for the benchmark's one-thread
    baseline) changes no result: route and layer are bit-identical on one
    thread and on all."""
    rng = np.random.default_rng(13)
    T, d, N_r, K, N_s, I = 50, 256, 8, 2, 1, 128
    u = _bf16(rng.standard_normal((T, d)))
    E = _bf16(rng.standard_normal((N_r, d)) / math.sqrt(d))
    routed, shared = _experts(rng, N_r, d, I, _bf16), _experts(rng, N_s, d, I, _bf16)
    n_all = R.set_threads(0)
    try:
        outs = []
        for n in (1, max(n_all, 2)):
            assert R.set_threads(n) == n
            r = R.route(u, E, np.zeros(N_r, np.float32), K)
            outs.append((r["idx"], r["key"], R.layer_forward(u, r["idx"], r["gate"], routed,
                                                             shared)))
    finally:
        R.set_threads(n_all)
    for a, b in zip(outs[0], outs[1]):
        np.testing.assert_array_equal(a, b)
