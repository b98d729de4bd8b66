"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test ties an oracle function to something the DeepSeek-V3 summary's
section 2 equations (h'-equation, affinity, g'-equation, bias rule) or plain
mathematics fix: a hand-derived example, brute force on tiny inputs, closed
forms, invariants, and special cases that reduce to an independent torch
float64 evaluation.  No GPU is used.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

HERE = os.path.dirname(__file__)


def _sigmoid(z):
    return 1.0 / (1.0 + math.exp(-z))


def _eval(expr):
    env = {"ln": math.log, "silu": lambda z: z * _sigmoid(z), "__builtins__": {}}
    return float(eval(expr, env))  # fixture expressions only (trusted, committed file)


def _rand_layer(rng, T, d, N_r, I, N_s, scale=1.0):
    u = rng.standard_normal((T, d))
    E = rng.standard_normal((N_r, d)) * scale / math.sqrt(d)
    routed = [(rng.standard_normal((I, d)) / math.sqrt(d),
               rng.standard_normal((I, d)) / math.sqrt(d),
               rng.standard_normal((d, I)) / math.sqrt(I)) for _ in range(N_r)]
    shared = [(rng.standard_normal((I, d)) / math.sqrt(d),
               rng.standard_normal((I, d)) / math.sqrt(d),
               rng.standard_normal((d, I)) / math.sqrt(I)) for _ in range(N_s)]
    return u, E, routed, shared


# --------------------------------------------------------------------------
# hand-derived example (tests/golden/handworked_layer.json)
# --------------------------------------------------------------------------

@pytest.fixture(scope="module")
def hand():
    with open(os.path.join(HERE, "golden", "handworked_layer.json")) as f:
        return json.load(f)


def _hand_arrays(h):
    u = np.array(h["u"], np.float64)
    E = np.array([[_eval(x) for x in row] for row in h["E_expr"]], np.float64)
    b = np.array(h["b"], np.float32)
    r = h["routed"]
    routed = [(np.array(r["W_gate"][i], float), np.array(r["W_up"][i], float),
               np.array(r["W_down"][i], float)) for i in range(h["N_r"])]
    s = h["shared"]
    shared = [(np.array(s["W_gate"][j], float), np.array(s["W_up"][j], float),
               np.array(s["W_down"][j], float)) for j in range(h["N_s"])]
    return u, E, b, routed, shared


def test_hand_example_routing(hand):
    u, E, b, _, _ = _hand_arrays(hand)
    r = O.route(u, E, b, hand["K"])
    assert r["idx"].tolist() == hand["expect"]["idx"]
    assert r["counts"].tolist() == hand["expect"]["counts"]
    want = np.array([[_eval(x) for x in row] for row in hand["expect"]["gate_expr"]])
    np.testing.assert_allclose(r["gate"], want, rtol=1e-6, atol=0)
    r0 = O.route(u, E, np.zeros(4, np.float32), hand["K"])
    assert r0["idx"].tolist() == hand["expect"]["idx_without_bias"]


def test_hand_example_layer(hand):
    u, E, b, routed, shared = _hand_arrays(hand)
    r = O.route(u, E, b, hand["K"])
    h = O.layer_forward(u, r["idx"], r["gate"], routed, shared)
    want = np.array([[_eval(x) for x in row] for row in hand["expect"]["h_expr"]])
    np.testing.assert_allclose(h, want, rtol=1e-6, atol=1e-7)


def test_hand_example_bias_update(hand):
    u, E, b, _, _ = _hand_arrays(hand)
    r = O.route(u, E, b, hand["K"])
    nb = O.bias_update(b, r["counts"], hand["T"], hand["K"])
    want = np.array([_eval(x) for x in hand["expect"]["b_after_expr"]], np.float32)
    np.testing.assert_array_equal(nb, want)


# --------------------------------------------------------------------------
# top-K against brute force
# --------------------------------------------------------------------------

def _brute_topk(key_row, K):
    """Enumerate every K-subset; keep the one whose keys dominate the rest,
    ties broken toward lower indices; order it by (key desc, index asc)."""
    n = len(key_row)
    best = None
    for sub in itertools.combinations(range(n), K):
        rest = [j for j in range(n) if j not in sub]
        ok = all((key_row[i] > key_row[j]) or (key_row[i] == key_row[j] and i < j)
                 for i in sub for j in rest)
        if ok:
            assert best is None, "two dominant subsets"
            best = sub
    return sorted(best, key=lambda i: (-key_row[i], i))


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce_random_and_ties(seed):
    rng = np.random.default_rng(seed)
    N_r = [4, 6, 8, 12, 16, 16][seed]
    K = [1, 2, 3, 4, 5, 16][seed]
    T = 40
    # quantised values produce many exact ties in s and in s + b
    s = (rng.integers(0, 5, size=(T, N_r)) / 8.0 + 0.25).astype(np.float32)
    b = (rng.integers(-2, 3, size=N_r) / 8.0).astype(np.float32)
    idx, key = O.biased_topk(s, b, K)
    for t in range(T):
        assert idx[t].tolist() == _brute_topk(key[t].tolist(), K)
        assert len(set(idx[t].tolist())) == K


def test_counts_and_distinct():
    rng = np.random.default_rng(7)
    u, E, _, _ = _rand_layer(rng, 300, 32, 16, 4, 0)
    b = rng.uniform(-0.01, 0.01, 16).astype(np.float32)
    r = O.route(u, E, b, 5)
    assert r["counts"].sum() == 300 * 5
    for row in r["idx"]:
        assert len(set(row.tolist())) == 5
    manual = np.zeros(16, int)
    for row in r["idx"]:
        for e in row:
            manual[e] += 1
    assert r["counts"].tolist() == manual.tolist()


# --------------------------------------------------------------------------
# gates
# --------------------------------------------------------------------------

def test_gates_sum_to_one():
    rng = np.random.default_rng(3)
    u, E, _, _ = _rand_layer(rng, 500, 64, 32, 4, 0, scale=3.0)
    b = rng.uniform(-0.1, 0.1, 32).astype(np.float32)
    for K in (1, 3, 8, 32):
        g = O.route(u, E, b, K)["gate"]
        err = np.abs(g.astype(np.float64).sum(axis=1) - 1.0)
        assert np.all(err <= 4 * np.finfo(np.float32).eps)
        assert np.all(g > 0)


def test_bias_never_changes_gate_values_zero_centroids():
    """E = 0: every s is Sigmoid(0) = 1/2, so any selection has gates 1/K,
    while the selection follows the largest b."""
    T, d, N_r = 16, 8, 10
    u = np.random.default_rng(0).standard_normal((T, d))
    E = np.zeros((N_r, d))
    b = np.array([0.01, -0.02, 0.05, 0.0, 0.03, -0.01, 0.02, 0.04, -0.03, 0.0], np.float32)
    for K in (1, 2, 4, 5):
        r = O.route(u, E, b, K)
        np.testing.assert_array_equal(r["gate"], np.float32(1.0 / K))
        want = sorted(range(N_r), key=lambda i: (-b[i], i))[:K]
        assert all(row.tolist() == want for row in r["idx"])


def test_same_selection_same_gates():
    """When two bias vectors select the same experts, gates are bit-identical."""
    rng = np.random.default_rng(11)
    u, E, _, _ = _rand_layer(rng, 200, 32, 16, 4, 0, scale=4.0)
    b1 = np.zeros(16, np.float32)
    b2 = np.full(16, 0.25, np.float32)          # a uniform shift never changes the order
    r1, r2 = O.route(u, E, b1, 4), O.route(u, E, b2, 4)
    same = np.all(np.sort(r1["idx"], 1) == np.sort(r2["idx"], 1), axis=1)
    assert same.all()
    np.testing.assert_array_equal(r1["gate"], r2["gate"])
    b3 = rng.uniform(-0.05, 0.05, 16).astype(np.float32)
    r3 = O.route(u, E, b3, 4)
    same3 = np.all(r1["idx"] == r3["idx"], axis=1)
    assert same3.any() and (~same3).any()
    np.testing.assert_array_equal(r1["gate"][same3], r3["gate"][same3])


# --------------------------------------------------------------------------
# layer special cases
# --------------------------------------------------------------------------

def test_dense_special_case_matches_torch():
    """K = N_r and b = 0: the layer is the dense sigmoid-weighted mixture
    u + sum_s FFN_s(u) + sum_i (s_i / sum_j s_j) FFN_i(u), evaluated here
    independently with torch float64 (sigmoid, einsum, silu)."""
    rng = np.random.default_rng(5)
    T, d, N_r, I, N_s = 24, 16, 6, 8, 2
    u, E, routed, shared = _rand_layer(rng, T, d, N_r, I, N_s)
    r = O.route(u, E, np.zeros(N_r, np.float32), N_r)
    got = O.layer_forward(u, r["idx"], r["gate"], routed, shared)

    tu, tE = torch.tensor(u), torch.tensor(E)
    s = torch.sigmoid(tu @ tE.T).float().double()        # s is stored as float32 (reading R3)
    w = s / s.sum(dim=1, keepdim=True)
    Wg = torch.tensor(np.stack([x[0] for x in routed]))
    Wu = torch.tensor(np.stack([x[1] for x in routed]))
    Wd = torch.tensor(np.stack([x[2] for x in routed]))
    hmid = torch.nn.functional.silu(torch.einsum("td,eid->tei", tu, Wg)) * torch.einsum("td,eid->tei", tu, Wu)
    y = torch.einsum("tei,edi->ted", hmid, Wd)
    want = tu + torch.einsum("te,ted->td", w, y)
    for (g_, u_, d_) in shared:
        hs = torch.nn.functional.silu(tu @ torch.tensor(g_).T) * (tu @ torch.tensor(u_).T)
        want = want + hs @ torch.tensor(d_).T
    # gates are float32 in the oracle, exact mixture weights in torch
    np.testing.assert_allclose(got, want.numpy(), rtol=2e-6, atol=2e-6)


def test_identical_experts():
    rng = np.random.default_rng(9)
    T, d, N_r, I = 30, 16, 8, 8
    u, E, routed, shared = _rand_layer(rng, T, d, N_r, I, 1)
    one = routed[0]
    same = [one] * N_r
    b = rng.uniform(-0.01, 0.01, N_r).astype(np.float32)
    r = O.route(u, E, b, 3)
    got = O.layer_forward(u, r["idx"], r["gate"], same, shared)
    want = u + O.swiglu_ffn(u, *shared[0]) + O.swiglu_ffn(u, *one)
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-6)


def test_zero_down_and_zero_input():
    rng = np.random.default_rng(2)
    T, d, N_r, I = 20, 8, 4, 4
    u, E, routed, shared = _rand_layer(rng, T, d, N_r, I, 1)
    r = O.route(u, E, np.zeros(N_r, np.float32), 2)
    zr = [(a, b_, np.zeros_like(c)) for (a, b_, c) in routed]
    zs = [(a, b_, np.zeros_like(c)) for (a, b_, c) in shared]
    np.testing.assert_array_equal(O.layer_forward(u, r["idx"], r["gate"], zr, zs), u)
    z = np.zeros_like(u)
    rz = O.route(z, E, np.zeros(N_r, np.float32), 2)
    np.testing.assert_array_equal(O.layer_forward(z, rz["idx"], rz["gate"], routed, shared), z)


def test_swiglu_against_torch_silu():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 8))
    Wg, Wu, Wd = rng.standard_normal((3, 8)), rng.standard_normal((3, 8)), rng.standard_normal((8, 3))
    tx = torch.tensor(x)
    want = (torch.nn.functional.silu(tx @ torch.tensor(Wg).T) * (tx @ torch.tensor(Wu).T)) @ torch.tensor(Wd).T
    np.testing.assert_allclose(O.swiglu_ffn(x, Wg, Wu, Wd), want.numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# permutation
# --------------------------------------------------------------------------

def test_permute_bijection_and_order():
    rng = np.random.default_rng(1)
    T, N_r, K = 97, 12, 3
    idx = np.stack([rng.choice(N_r, K, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, perm_src, inv = O.permute_indices(idx, N_r)
    counts = np.bincount(idx.reshape(-1), minlength=N_r)
    assert offsets[0] == 0 and offsets[-1] == T * K
    np.testing.assert_array_equal(np.diff(offsets), counts)
    assert sorted(inv.reshape(-1).tolist()) == list(range(T * K))
    for t in range(T):
        for k in range(K):
            p = inv[t, k]
            assert perm_src[p] == t
            e = idx[t, k]
            assert offsets[e] <= p < offsets[e + 1]
    for e in range(N_r):
        seg = perm_src[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_permute_with_empty_experts():
    idx = np.array([[0, 3], [3, 0], [0, 3]], np.int32)
    offsets, perm_src, inv = O.permute_indices(idx, 5)
    assert offsets.tolist() == [0, 3, 3, 3, 6, 6]
    assert perm_src.tolist() == [0, 1, 2, 0, 1, 2]
    assert inv.tolist() == [[0, 3], [4, 1], [2, 5]]


# --------------------------------------------------------------------------
# bias update sign rule
# --------------------------------------------------------------------------

def test_bias_sign_rule():
    N_r, T, K = 8, 10, 4          # mean load T*K/N_r = 5
    counts = np.array([5, 6, 4, 0, 15, 5, 3, 2], np.int32)
    assert counts.sum() == T * K
    b = np.array([0.0, 0.1, -0.1, 0.5, 0.0, -0.3, 0.02, 1.0], np.float32)
    nb = O.bias_update(b, counts, T, K)
    g = np.float32(0.001)
    want = np.array([b[0], b[1] - g, b[2] + g, b[3] + g, b[4] - g, b[5], b[6] + g, b[7] + g], np.float32)
    np.testing.assert_array_equal(nb, want)
    under, over = int((counts * N_r < T * K).sum()), int((counts * N_r > T * K).sum())
    assert abs(float(nb.astype(np.float64).sum() - b.astype(np.float64).sum())
               - 0.001 * (under - over)) < 1e-6


def test_bias_update_mean_is_not_rounded():
    """Mean load 10*3/4 = 7.5: a load of 7 is under, 8 is over (integer compare)."""
    nb = O.bias_update(np.zeros(4, np.float32), np.array([7, 8, 7, 8]), 10, 3)
    np.testing.assert_array_equal(nb, np.array([0.001, -0.001, 0.001, -0.001], np.float32))


# --------------------------------------------------------------------------
# FP8 recipe
# --------------------------------------------------------------------------

def _all_e4m3_values():
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue                      # the NaN code of E4M3
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.add(v)
            vals.add(-v)
    return np.array(sorted(vals))


def test_e4m3_grid():
    v = _all_e4m3_values()
    assert v.max() == 448.0 and len(v) == 253            # +-0 collapse into one value
    np.testing.assert_array_equal(O.e4m3_round(v), v)    # representable values round-trip


def test_e4m3_matches_torch_rne():
    """Within the finite range, rounding must equal torch's float8_e4m3fn cast
    (a library round-to-nearest-even), including every exact midpoint."""
    v = _all_e4m3_values()
    pos = v[v >= 0]
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.uniform(-460, 460, 20000), rng.standard_normal(20000) * 1e-2,
                           rng.standard_normal(20000) * 1e-3])
    x = np.concatenate([mids, -mids, rand, pos * 1.0000001, pos * 0.9999999]).astype(np.float32)
    x = x[np.abs(x) < 464.0]
    want = torch.tensor(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_round(x), want)


def test_e4m3_saturates():
    np.testing.assert_array_equal(O.e4m3_round(np.array([464.0, 500.0, 1e6, -1e9])),
                                  [448.0, 448.0, 448.0, -448.0])


def test_quant_1x128_properties():
    rng = np.random.default_rng(8)
    X = (rng.standard_normal((6, 384)) * np.array([1, 50, 1e-3])[np.arange(384) // 128]).astype(np.float32)
    X[5, 128:256] = 0.0
    q, sc = O.quant_1x128(X)
    assert sc.shape == (6, 3) and sc[5, 1] == 1.0
    np.testing.assert_array_equal(q[5, 128:256], 0.0)
    for r in range(6):
        for t in range(3):
            blk = X[r, t * 128:(t + 1) * 128]
            if np.abs(blk).max() == 0:
                continue
            j = np.argmax(np.abs(blk))
            assert abs(q[r, t * 128 + j]) == 448.0              # amax maps to +-448
            assert np.all(np.abs(q[r, t * 128:(t + 1) * 128]) <= 448.0)
    deq = q * np.repeat(sc, 128, axis=1)
    rel = np.abs(deq - X) / np.repeat(np.abs(X).reshape(6, 3, 128).max(2), 128, axis=1).clip(1e-30)
    assert rel.max() <= 2.0 ** -4 + 1e-7                   # half an E4M3 ulp at the top binade


def test_quant_128x128_blocks():
    rng = np.random.default_rng(9)
    W = rng.standard_normal((256, 384)).astype(np.float32)
    W[:128, 128:256] *= 100
    q, sc = O.quant_128x128(W)
    assert sc.shape == (2, 3)
    np.testing.assert_allclose(sc[0, 1], np.abs(W[:128, 128:256]).max() / np.float32(448), rtol=1e-7)
    assert np.abs(q).max() == 448.0


def test_promoted_gemm_unit_scales_is_plain_sum():
    rng = np.random.default_rng(10)
    v = _all_e4m3_values()
    qa = rng.choice(v, size=(7, 256))
    qw = rng.choice(v, size=(128, 256))
    got = O.fp8_promoted_gemm(qa, np.ones((7, 2), np.float32), qw, np.ones((1, 2), np.float32))
    want = np.array([[sum(qa[r, k] * qw[n, k] for k in range(256)) for n in range(128)] for r in range(7)])
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-9)


def test_promoted_gemm_scales_per_block():
    """Each 128-wide K block carries its own scale pair: scaling one block's
    activation scale by 2 adds exactly that block's partial once more."""
    rng = np.random.default_rng(12)
    v = _all_e4m3_values()
    qa = rng.choice(v[np.abs(v) < 8], size=(3, 256))
    qw = rng.choice(v[np.abs(v) < 8], size=(128, 256))
    sa = np.ones((3, 2), np.float32)
    sw = np.ones((1, 2), np.float32)
    base = O.fp8_promoted_gemm(qa, sa, qw, sw)
    sa2 = sa.copy()
    sa2[:, 1] = 2
    got = O.fp8_promoted_gemm(qa, sa2, qw, sw)
    np.testing.assert_allclose(got - base, qa[:, 128:] @ qw[:, 128:].T, rtol=1e-12, atol=1e-9)


def test_fp8_ffn_close_to_exact():
    """The FP8 FFN stays within the recipe's expected error of the exact
    float64 FFN.  E4M3 keeps 3 mantissa bits (relative rounding error up to
    2^-4, about 2.5 % rms); four quantised operands along the SwiGLU chain
    compound to about 6.5 % rms, so the bound is 9 % rms and 15 % of the
    output's maximum.  A dropped or misapplied scale misses it by orders."""
    rng = np.random.default_rng(13)
    d, I = 256, 128
    x = rng.standard_normal((16, d)).astype(np.float32)
    Wg, Wu = rng.standard_normal((I, d)) / 16, rng.standard_normal((I, d)) / 16
    Wd = rng.standard_normal((d, I)) / math.sqrt(I)
    Wq = O.quantise_expert(Wg.astype(np.float32), Wu.astype(np.float32), Wd.astype(np.float32))
    got = O.fp8_swiglu_ffn(x, Wq)
    want = O.swiglu_ffn(x, Wg, Wu, Wd)
    rms = np.sqrt(((got - want) ** 2).mean() / (want ** 2).mean())
    assert rms <= 0.09
    assert np.abs(got - want).max() <= 0.15 * np.abs(want).max()


# --------------------------------------------------------------------------
# group-limited routing
# --------------------------------------------------------------------------

def _brute_grouped(key_row, K, G, M):
    """Enumerate every choice of M groups (score = best key, ties to lower
    group index as a dominant set), then the best K keys inside them."""
    n = len(key_row)
    gs = n // G
    gscore = [max(key_row[g * gs:(g + 1) * gs]) for g in range(G)]
    best = None
    for gsub in itertools.combinations(range(G), M):
        rest = [g for g in range(G) if g not in gsub]
        if all(gscore[a] > gscore[c] or (gscore[a] == gscore[c] and a < c)
               for a in gsub for c in rest):
            best = gsub
    allowed = [i for i in range(n) if i // gs in best]
    return sorted(allowed, key=lambda i: (-key_row[i], i))[:K]


@pytest.mark.parametrize("seed", range(4))
def test_grouped_topk_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    N_r, G, M, K = [(16, 4, 2, 3), (12, 3, 1, 4), (16, 8, 3, 5), (8, 2, 2, 8)][seed]
    s = (rng.integers(0, 6, size=(50, N_r)) / 8.0 + 0.2).astype(np.float32)
    b = (rng.integers(-2, 3, size=N_r) / 16.0).astype(np.float32)
    idx, key = O.grouped_topk(s, b, K, G, M)
    for t in range(50):
        assert idx[t].tolist() == _brute_grouped(key[t].tolist(), K, G, M)
        assert len({int(e) // (N_r // G) for e in idx[t]}) <= M


def test_grouped_topk_special_cases():
    rng = np.random.default_rng(5)
    s = rng.uniform(0, 1, (200, 32)).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, 32).astype(np.float32)
    plain, _ = O.biased_topk(s, b, 6)
    for G in (1, 2, 4, 8):                       # keeping every group is no limit
        np.testing.assert_array_equal(O.grouped_topk(s, b, 6, G, G)[0], plain)
    idx, key = O.grouped_topk(s, b, 6, 8, 2)
    assert np.all(idx[:, 0] == np.argmax(key, axis=1))   # the best expert's group always survives


# --------------------------------------------------------------------------
# near-tie margins used by the routing comparison
# --------------------------------------------------------------------------

def test_topk_margins_hand_worked():
    """Worked by hand: row 0 sorts to 0.80, 0.80, 0.79 | 0.50 ...: the K-th
    (3rd) key 0.79 minus the next key 0.50, and a zero gap between the two
    equal selected keys; row 1 sorts to 0.9, 0.7, 0.65 | 0.6: gaps 0.05 and
    min(0.2, 0.05).  K = N_r has no next key (infinite gap), K = 1 has no
    adjacent selected pair (infinite gap)."""
    f = np.float32
    key = np.array([[0.50, 0.80, 0.30, 0.80, 0.79, 0.10],
                    [0.90, 0.60, 0.70, 0.65, 0.20, 0.10]], np.float32)
    idx, _ = O.biased_topk(key, np.zeros(6, np.float32), 3)
    assert idx.tolist() == [[1, 3, 4], [0, 2, 3]]
    sel, inner = O.topk_margins(key, idx)
    assert sel[0] == float(f(0.79)) - float(f(0.50))
    assert sel[1] == float(f(0.65)) - float(f(0.60))
    assert inner[0] == 0.0
    assert inner[1] == float(f(0.70)) - float(f(0.65))
    full, _ = O.biased_topk(key, np.zeros(6, np.float32), 6)
    sel6, inner6 = O.topk_margins(key, full)
    assert np.all(np.isinf(sel6)) and inner6[0] == 0.0
    one, _ = O.biased_topk(key, np.zeros(6, np.float32), 1)
    sel1, inner1 = O.topk_margins(key, one)
    assert sel1[0] == 0.0 and sel1[1] == float(f(0.90)) - float(f(0.70))
    assert np.all(np.isinf(inner1))


# --------------------------------------------------------------------------
# the layer under the FP8 recipe
# --------------------------------------------------------------------------

def _fp8_layer_case(seed, T=12, d=256, N_r=5, I=128, N_s=1):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((T, d)).astype(np.float32).astype(np.float64)
    E = rng.standard_normal((N_r, d)) / math.sqrt(d)

    def q():
        return O.quantise_expert((rng.standard_normal((I, d)) / math.sqrt(d)).astype(np.float32),
                                 (rng.standard_normal((I, d)) / math.sqrt(d)).astype(np.float32),
                                 (rng.standard_normal((d, I)) / math.sqrt(I)).astype(np.float32))
    return u, E, [q() for _ in range(N_r)], [q() for _ in range(N_s)]


def test_fp8_layer_identical_experts():
    """All routed experts equal: the gates sum to 1, so the routed term is one
    FP8 FFN whatever the routing; the shared term enters with weight 1."""
    u, E, routed, shared = _fp8_layer_case(21)
    r = O.route(u, E, np.zeros(len(routed), np.float32), 3)
    got = O.layer_forward_fp8(u, r["idx"], r["gate"], [routed[0]] * len(routed), shared)
    want = u + O.fp8_swiglu_ffn(u, shared[0]) + O.fp8_swiglu_ffn(u, routed[0])
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-6)


def test_fp8_layer_zero_down_and_zero_input():
    """W_down = 0 quantises to zero codes with unit scales: h' = u exactly;
    u = 0 quantises to zero codes: every FFN is 0 and h' = 0 exactly."""
    u, E, routed, shared = _fp8_layer_case(22)
    zero = lambda Wq: {**Wq, "down": (np.zeros_like(Wq["down"][0]),
                                      O.tile_scale(np.zeros_like(Wq["down"][1])))}
    r = O.route(u, E, np.zeros(len(routed), np.float32), 2)
    got = O.layer_forward_fp8(u, r["idx"], r["gate"], [zero(w) for w in routed],
                              [zero(w) for w in shared])
    np.testing.assert_array_equal(got, u)
    z = np.zeros_like(u)
    rz = O.route(z, E, np.zeros(len(routed), np.float32), 2)
    np.testing.assert_array_equal(O.layer_forward_fp8(z, rz["idx"], rz["gate"], routed, shared), z)


def test_fp8_layer_dense_mixture():
    """K = N_r, b = 0: the FP8 layer is u + sum_s FFN8_s(u) + sum_i (s_i / sum_j
    s_j) FFN8_i(u), written here as a plain loop over every expert on every
    token (activation scales are per row, so each row quantises alike in any
    batch).  Catches a gate applied to the wrong slot or a dropped term."""
    u, E, routed, shared = _fp8_layer_case(23, N_s=2)
    N_r = len(routed)
    r = O.route(u, E, np.zeros(N_r, np.float32), N_r)
    got = O.layer_forward_fp8(u, r["idx"], r["gate"], routed, shared)
    s = (1.0 / (1.0 + np.exp(-(u @ E.T)))).astype(np.float32).astype(np.float64)
    w = s / s.sum(axis=1, keepdims=True)
    want = u.copy()
    for Wq in shared:
        want += O.fp8_swiglu_ffn(u, Wq)
    for i in range(N_r):
        want += w[:, i:i + 1] * O.fp8_swiglu_ffn(u, routed[i])
    np.testing.assert_allclose(got, want, rtol=2e-6, atol=2e-6)


def _e4m3_nearest(x):
    """Brute force: the nearest of the 253 finite E4M3 values (saturating),
    ties to the code with the even mantissa, found by search over the table."""
    vals, even = [], []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            for sgn in (1.0, -1.0):
                vals.append(sgn * v)
                even.append(m % 2 == 0)
    vals, even = np.array(vals), np.array(even)
    x = np.asarray(x, np.float64)
    dist = np.abs(x.reshape(-1, 1) - vals[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    pick = np.where(cand & even[None, :], 1, 0) + np.where(cand, 1, 0)
    return vals[np.argmax(pick, axis=1)].reshape(x.shape)


def _fp8_ffn_brute(x, Wg, Wu, Wd, h_round):
    """The FP8 SwiGLU FFN of reading R6 with scalar loops on a tiny case:
    1x128 activation tiles and 128x128 weight blocks with float32 scales
    amax/448, each 128-deep partial sum times its two scales, h formed by
    h_round (float32 per R6) and re-quantised 1x128."""
    f32 = np.float32

    def quant(M, rb, cb):
        M = np.asarray(M, np.float32)
        q = np.zeros(M.shape)
        sc = np.zeros((M.shape[0] // rb, M.shape[1] // cb), np.float32)
        for i in range(sc.shape[0]):
            for j in range(sc.shape[1]):
                blk = M[i * rb:(i + 1) * rb, j * cb:(j + 1) * cb]
                amax = f32(np.abs(blk).max())
                s = f32(1.0) if amax == 0 else f32(amax / f32(448.0))
                sc[i, j] = s
                q[i * rb:(i + 1) * rb, j * cb:(j + 1) * cb] = _e4m3_nearest(blk / s)
        return q, sc

    def gemm(qa, sa, qw, sw):
        R, Kd = qa.shape
        out = np.zeros((R, qw.shape[0]))
        for r in range(R):
            for n in range(qw.shape[0]):
                acc = 0.0
                for kb in range(Kd // 128):
                    part = 0.0
                    for k in range(kb * 128, kb * 128 + 128):
                        part += qa[r, k] * qw[n, k]
                    acc += part * float(sa[r, kb]) * float(sw[n // 128, kb])
                out[r, n] = acc
        return out

    qx, sx = quant(x, 1, 128)
    g = gemm(qx, sx, *quant(Wg, 128, 128))
    v = gemm(qx, sx, *quant(Wu, 128, 128))
    h = np.array([[h_round(gg / (1.0 + math.exp(-gg)) * vv) for gg, vv in zip(gr, vr)]
                  for gr, vr in zip(g, v)])
    qh, sh = quant(h, 1, 128)
    return gemm(qh, sh, *quant(Wd, 128, 128))


def test_fp8_ffn_bruteforce_tiny():
    """fp8_swiglu_ffn equals the brute-force evaluation of reading R6 (own
    E4M3 table search, scalar loops) on a 3-row case with two 128-deep K
    blocks, and the case is sensitive to the precision of h: rounding h to
    bf16 instead of float32 before its re-quantisation changes the result."""
    rng = np.random.default_rng(31)
    d, I = 256, 128
    x = rng.standard_normal((3, d)).astype(np.float32)
    x[1, 7] = 40.0                                        # an outlier in one tile
    Wg = (rng.standard_normal((I, d)) / 16).astype(np.float32)
    Wu = (rng.standard_normal((I, d)) / 16).astype(np.float32)
    Wd = (rng.standard_normal((d, I)) / math.sqrt(I)).astype(np.float32)
    got = O.fp8_swiglu_ffn(x, O.quantise_expert(Wg, Wu, Wd))
    want = _fp8_ffn_brute(x, Wg, Wu, Wd, lambda z: float(np.float32(z)))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    bf16 = lambda z: float(torch.tensor(z, dtype=torch.float32).to(torch.bfloat16).float())
    other = _fp8_ffn_brute(x, Wg, Wu, Wd, bf16)
    assert np.abs(other - want).max() > 1e-6 * np.abs(want).max()
