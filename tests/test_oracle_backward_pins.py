"""Pins for the backward oracle (oracle/moe_backward.py), each independent of
the chain-rule formulas it checks:

  * central finite differences of the forward oracle (every gradient entry of
    a tiny layer);
  * torch float64 autograd of a torch evaluation of the forward, at a larger
    size;
  * closed forms: W_down = 0 leaves only the residual in du and gives dE = 0;
    identical experts with K = N_r make h' independent of s, so dE = 0;
  * the gate invariant: scaling every selected s by one factor leaves g
    unchanged, so sum_k ds_k s_k = 0;
  * FP8 backward: the Wgrad quantiser equals the pinned forward quantiser on
    the transpose, its blocks follow the groups, promoted Wgrad/Dgrad with
    unit scales are plain products, scales act per block row and column, and
    the FP8 expert and layer backward stay within E4M3's error of the exact one.
"""
import numpy as np
import pytest
import torch

from oracle import moe_backward as B
from oracle import moe_oracle as O


def _problem(T, d, N_r, K, N_s, I, seed):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((T, d))
    E = rng.standard_normal((N_r, d)) / np.sqrt(d)
    routed = [(rng.standard_normal((I, d)) / np.sqrt(d), rng.standard_normal((I, d)) / np.sqrt(d),
               rng.standard_normal((d, I)) / np.sqrt(I)) for _ in range(N_r)]
    shared = [(rng.standard_normal((I, d)) / np.sqrt(d), rng.standard_normal((I, d)) / np.sqrt(d),
               rng.standard_normal((d, I)) / np.sqrt(I)) for _ in range(N_s)]
    b = rng.uniform(-0.05, 0.05, N_r).astype(np.float32)
    idx = O.route(u, E, b, K)["idx"]
    dh = rng.standard_normal((T, d))
    return u, E, routed, shared, idx, dh


def _objective(u, E, routed, shared, idx, dh):
    """L = <dh, h'> with the selection idx held fixed and g from float64 s."""
    s = 1.0 / (1.0 + np.exp(-(u @ E.T)))
    sel = np.take_along_axis(s, idx, axis=1)
    g = sel / sel.sum(axis=1, keepdims=True)
    return float(np.sum(dh * O.layer_forward(u, idx, g, routed, shared)))


def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def test_backward_matches_finite_differences():
    u, E, routed, shared, idx, dh = _problem(T=4, d=6, N_r=5, K=2, N_s=1, I=3, seed=11)
    got = B.layer_backward(u, E, idx, routed, shared, dh)
    f = lambda: _objective(u, E, routed, shared, idx, dh)
    np.testing.assert_allclose(got["du"], _fd(f, u), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(got["dE"], _fd(f, E), rtol=1e-6, atol=1e-8)
    for e in range(len(routed)):
        for m, W in enumerate(routed[e]):
            want = _fd(f, W)
            have = got["routed"][e][m] if e in got["routed"] else np.zeros_like(W)
            np.testing.assert_allclose(have, want, rtol=1e-6, atol=1e-8, err_msg=f"expert {e} m {m}")
    for m, W in enumerate(shared[0]):
        np.testing.assert_allclose(got["shared"][0][m], _fd(f, W), rtol=1e-6, atol=1e-8)


def test_backward_matches_torch_autograd():
    T, d, N_r, K, N_s, I = 48, 32, 8, 3, 2, 16
    u, E, routed, shared, idx, dh = _problem(T, d, N_r, K, N_s, I, seed=12)
    got = B.layer_backward(u, E, idx, routed, shared, dh)

    tt = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    U, Et = tt(u), tt(E)
    R = [[tt(w) for w in ex] for ex in routed]
    S = [[tt(w) for w in ex] for ex in shared]

    def ffn(x, Wg, Wu, Wd):
        return torch.nn.functional.linear(
            torch.nn.functional.silu(torch.nn.functional.linear(x, Wg))
            * torch.nn.functional.linear(x, Wu), Wd)

    it = torch.tensor(idx, dtype=torch.long)
    s = torch.sigmoid(U @ Et.T)
    sel = torch.gather(s, 1, it)
    g = sel / sel.sum(1, keepdim=True)
    h = U.clone()
    for ex in S:
        h = h + ffn(U, *ex)
    for e in range(N_r):
        # dense evaluation, masked: every token through every expert
        w = (g * (it == e)).sum(1, keepdim=True)
        h = h + w * ffn(U, *R[e])
    (h * torch.tensor(dh)).sum().backward()

    np.testing.assert_allclose(got["du"], U.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(got["dE"], Et.grad.numpy(), rtol=1e-10, atol=1e-12)
    for e in range(N_r):
        for m in range(3):
            have = got["routed"][e][m] if e in got["routed"] else np.zeros_like(routed[e][m])
            np.testing.assert_allclose(have, R[e][m].grad.numpy(), rtol=1e-10, atol=1e-12)
    for j in range(N_s):
        for m in range(3):
            np.testing.assert_allclose(got["shared"][j][m], S[j][m].grad.numpy(),
                                       rtol=1e-10, atol=1e-12)


def test_zero_down_projection_leaves_residual_only():
    u, E, routed, shared, idx, dh = _problem(T=16, d=8, N_r=6, K=2, N_s=1, I=4, seed=13)
    routed = [(g, v, np.zeros_like(w)) for g, v, w in routed]
    shared = [(g, v, np.zeros_like(w)) for g, v, w in shared]
    got = B.layer_backward(u, E, idx, routed, shared, dh)
    np.testing.assert_array_equal(got["du"], dh)
    assert not got["dE"].any()
    assert not got["d_gate"].any()
    for e, (dWg, dWu, dWd) in got["routed"].items():
        assert not dWg.any() and not dWu.any()
        assert np.abs(dWd).max() > 0          # dW_down = dy^T h still flows


def test_identical_experts_dense_routing_has_no_router_gradient():
    u, E, routed, shared, _, dh = _problem(T=10, d=8, N_r=4, K=4, N_s=0, I=5, seed=14)
    routed = [routed[0]] * 4
    idx = np.tile(np.arange(4, dtype=np.int32), (10, 1))
    got = B.layer_backward(u, E, idx, routed, [], dh)
    assert np.abs(got["dE"]).max() < 1e-13
    assert np.abs(got["d_logit"]).max() < 1e-13
    # and du is the residual plus one expert's input gradient
    dx = B.swiglu_ffn_backward(u, *routed[0], dh)[0]
    np.testing.assert_allclose(got["du"], dh + dx, rtol=1e-12, atol=1e-12)


def test_gate_gradient_orthogonal_to_s():
    rng = np.random.default_rng(15)
    s = rng.uniform(0.05, 0.95, (20, 8))
    dg = rng.standard_normal((20, 8))
    ds = B.gate_backward(s, dg)
    np.testing.assert_allclose(np.sum(ds * s, axis=1), 0.0, atol=1e-13)


@pytest.mark.parametrize("z", [-30.0, -2.0, 0.0, 0.5, 3.0, 30.0])
def test_silu_grad_is_derivative(z):
    eps = 1e-6
    fd = (O.silu(z + eps) - O.silu(z - eps)) / (2 * eps)
    assert abs(B.silu_grad(z) - fd) < 1e-8


# ---------------------------------------------------------------- FP8 backward (reading B5)

def test_quant_128x1_matches_transposed_1x128():
    """One group of whole 128-row blocks: the Wgrad quantiser is the forward's
    1x128 quantiser applied to the transpose (an independent, pinned routine)."""
    rng = np.random.default_rng(21)
    X = (rng.standard_normal((256, 384)) * rng.uniform(0.1, 10, 384)[None, :]).astype(np.float32)
    X[:128, 5] = 0.0                                   # an all-zero column block -> scale 1
    q, sc, blocks = B.quant_128x1_grouped(X, [0, 256])
    qt, sct = O.quant_1x128(X.T)
    np.testing.assert_array_equal(q, qt.T)
    np.testing.assert_array_equal(sc, sct.T)
    assert blocks == [(0, 0, 128), (0, 128, 256)]
    assert sc[0, 5] == 1.0


def test_quant_128x1_grouped_blocks_follow_groups():
    """Blocks start at every group's first row, the last one of a group may be
    short, empty groups have none; each scale is its block's column amax/448."""
    rng = np.random.default_rng(22)
    sizes = [0, 3, 128, 130, 0, 257]
    off = np.concatenate([[0], np.cumsum(sizes)])
    X = rng.standard_normal((off[-1], 128)).astype(np.float32)
    q, sc, blocks = B.quant_128x1_grouped(X, off)
    want = [(1, 0, 3), (2, 3, 131), (3, 131, 259), (3, 259, 261),
            (5, 261, 389), (5, 389, 517), (5, 517, 518)]
    assert blocks == want
    for i, (g, r0, r1) in enumerate(blocks):
        amax = np.abs(X[r0:r1]).max(axis=0)
        np.testing.assert_array_equal(sc[i], (amax / np.float32(448)).astype(np.float32))
        # the largest element of every column maps to +-448 exactly
        col = np.argmax(np.abs(X[r0:r1]), axis=0)
        np.testing.assert_array_equal(np.abs(q[r0:r1][col, np.arange(128)]), 448.0)


def test_fp8_wgrad_and_dgrad_with_unit_scales_are_plain_products():
    rng = np.random.default_rng(23)
    qa = O.e4m3_round(rng.standard_normal((300, 128)) * 8)
    qb = O.e4m3_round(rng.standard_normal((300, 256)) * 8)
    blocks = [(0, 0, 100), (1, 100, 228), (1, 228, 300)]
    ones_a, ones_b = np.ones((3, 128), np.float32), np.ones((3, 256), np.float32)
    got = B.fp8_wgrad(qa, ones_a, qb, ones_b, blocks, 2)
    np.testing.assert_array_equal(got[0], qa[:100].T @ qb[:100])
    np.testing.assert_array_equal(got[1], qa[100:].T @ qb[100:])
    qdy = O.e4m3_round(rng.standard_normal((7, 256)) * 8)
    qW = O.e4m3_round(rng.standard_normal((256, 384)) * 8)
    got = B.fp8_dgrad(qdy, np.ones((7, 2), np.float32), qW, np.ones((2, 3), np.float32))
    np.testing.assert_array_equal(got, qdy @ qW)


def test_fp8_wgrad_scales_apply_per_block_row_and_column():
    rng = np.random.default_rng(24)
    qa = O.e4m3_round(rng.standard_normal((200, 128)))
    qb = O.e4m3_round(rng.standard_normal((200, 128)))
    sa = rng.uniform(0.5, 2, (2, 128)).astype(np.float32)
    sb = rng.uniform(0.5, 2, (2, 128)).astype(np.float32)
    blocks = [(0, 0, 128), (0, 128, 200)]
    got = B.fp8_wgrad(qa, sa, qb, sb, blocks, 1)[0]
    want = ((qa[:128] * sa[0]).T @ (qb[:128] * sb[0])) + ((qa[128:] * sa[1]).T @ (qb[128:] * sb[1]))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_fp8_ffn_backward_close_to_exact():
    """The FP8 backward of one expert stays within the error E4M3 quantisation
    of every GEMM input implies (3-bit mantissa: relative step 2^-3..2^-4, so a
    few percent per quantised operand, compounded over two chained GEMMs)."""
    rng = np.random.default_rng(25)
    R, d, I = 300, 256, 256
    x = rng.standard_normal((R, d)).astype(np.float32)
    Wg = (rng.standard_normal((I, d)) / np.sqrt(d)).astype(np.float32)
    Wu = (rng.standard_normal((I, d)) / np.sqrt(d)).astype(np.float32)
    Wd = (rng.standard_normal((d, I)) / np.sqrt(I)).astype(np.float32)
    dy = (rng.standard_normal((R, d)) * 0.05).astype(np.float32)
    got = B.fp8_swiglu_ffn_backward(x, O.quantise_expert(Wg, Wu, Wd), dy)
    want = B.swiglu_ffn_backward(x, Wg, Wu, Wd, dy)
    for name, a, b in zip(["dx", "dW_gate", "dW_up", "dW_down"], got, want[:4]):
        rel = np.sqrt(np.mean((a - b) ** 2) / np.mean(b ** 2))
        assert rel < 0.12, (name, rel)
        assert rel > 1e-3, (name, rel)      # the quantisation really happened


def test_fp8_layer_backward_close_to_exact():
    u, E, routed, shared, idx, dh = _problem(T=40, d=256, N_r=4, K=2, N_s=1, I=128, seed=26)
    rq = [O.quantise_expert(*ex) for ex in routed]
    sq = [O.quantise_expert(*ex) for ex in shared]
    got = B.layer_backward_fp8(u, E, idx, rq, sq, dh)
    want = B.layer_backward(u, E, idx, routed, shared, dh)
    for key in ("du", "dE", "d_gate"):
        a, b = got[key], want[key]
        rel = np.sqrt(np.mean((a - b) ** 2) / np.mean(b ** 2))
        assert rel < 0.12, (key, rel)
    for e in got["routed"]:
        for a, b in zip(got["routed"][e], want["routed"][e]):
            assert np.sqrt(np.mean((a - b) ** 2) / np.mean(b ** 2)) < 0.12
