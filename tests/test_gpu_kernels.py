"""Per-call parity of libmoe's kernels against the CPU oracle, through the
C ABI, at sizes that span several tiles with ragged tails, plus edge cases.
Integer and index outputs must match bit for bit; floating-point outputs
within the tolerances of tests/harness.py."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_60_b200 as moe
from oracle import moe_backward as B
from oracle import moe_oracle as O
from tests.harness import (GATE_TOL, TOL, LazyExperts, assert_close, check_routing, f64,
                           TIE_GAP, grouped_reference)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _randn(shape, g, std=1.0, dtype=torch.bfloat16):
    return (torch.randn(*shape, generator=g, device=DEV) * std).to(dtype)


def _ws(n):
    return torch.empty(max(n, 256), dtype=torch.uint8, device=DEV)


def _route(u, E, b, K):
    T, N_r = u.shape[0], E.shape[0]
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    gate = torch.empty(T, K, dtype=torch.float32, device=DEV)
    counts = torch.full((N_r,), -7, dtype=torch.int32, device=DEV)
    moe.moe_route(u, E, b, K, idx, gate, counts, _ws(moe.moe_route_workspace_size(T, N_r)))
    torch.cuda.synchronize()
    return idx, gate, counts


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("T,d,N_r,K,dt", [
    (1000, 512, 64, 6, torch.bfloat16),     # tensor-core logits, BN = 64
    (517, 1024, 256, 8, torch.bfloat16),    # BN = 256, ragged last tile
    (300, 256, 128, 8, torch.bfloat16),     # BN = 128
    (333, 256, 16, 4, torch.float32),       # CUDA-core logits
    (257, 192, 32, 3, torch.float32),
    (200, 128, 16, 4, torch.bfloat16),      # N_r not a multiple of 64 -> CUDA-core logits
    (64, 128, 64, 1, torch.bfloat16),       # K = 1
    (50, 128, 64, 64, torch.bfloat16),      # K = N_r
    (1, 128, 64, 6, torch.bfloat16),        # one token
    (20000, 256, 256, 8, torch.bfloat16),   # more 256-token tiles than CTA pairs: tile loop
    (700, 256, 96, 16, torch.bfloat16),     # N_r = 96, K = 16
    (300, 256, 1024, 8, torch.bfloat16),    # N_r = 1024, the most the library takes
])
def test_route_matches_oracle(T, d, N_r, K, dt):
    g = _gen(T * 31 + d)
    u = _randn((T, d), g, 1.0, dt)
    E = _randn((N_r, d), g, d ** -0.5, dt)
    b = ((torch.rand(N_r, generator=g, device=DEV) * 2 - 1) * 0.01).float()
    idx, gate, counts = _route(u, E, b, K)
    ref = O.route(f64(u), f64(E), b.cpu().numpy(), K)
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy(), ref, K,
                  gate_tol=GATE_TOL["f32" if dt == torch.float32 else "bf16"])
    np.testing.assert_allclose(gate.double().sum(1).cpu().numpy(), 1.0, atol=4e-7)
    assert moe.moe_device_status() == 0


@pytest.mark.parametrize("T,d,N_r,K,G,M", [
    (1000, 512, 256, 8, 8, 4), (333, 256, 64, 6, 4, 2), (200, 128, 64, 4, 16, 1),
    (300, 256, 128, 8, 8, 8),    # keeping every group: same as no limit
    (20000, 256, 256, 8, 8, 4),  # tile loop of the fused router
])
def test_route_grouped_matches_oracle(T, d, N_r, K, G, M):
    g = _gen(T + G * 7)
    u = _randn((T, d), g)
    E = _randn((N_r, d), g, d ** -0.5)
    b = ((torch.rand(N_r, generator=g, device=DEV) * 2 - 1) * 0.01).float()
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    gate = torch.empty(T, K, dtype=torch.float32, device=DEV)
    counts = torch.empty(N_r, dtype=torch.int32, device=DEV)
    moe.moe_route_grouped(u, E, b, K, G, M, idx, gate, counts,
                          _ws(moe.moe_route_workspace_size(T, N_r)))
    torch.cuda.synchronize()
    ref = O.route_grouped(f64(u), f64(E), b.cpu().numpy(), K, G, M)
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy(),
                  grouped_reference(ref, K, G, M), K, gate_tol=GATE_TOL["bf16"])
    gsz = N_r // G
    assert max(len(set((r // gsz).tolist())) for r in idx.cpu().numpy()) <= M


def _listed_tokens(ws, T, N_r):
    """Tokens the router sent to its float64 tie-break (white-box: the count
    is the first word after the float32 logits in the router workspace)."""
    off = (T * N_r * 4 + 255) // 256 * 256
    return int(ws[off:off + 4].view(torch.int32)[0])


def test_route_v3_width_float64_tie_break():
    """d = 7168 (V3): float32 tensor-core logits are off by a few 1e-6, so
    some tokens are decided within the refine gap; routing must still match
    the float64 oracle."""
    T, d, N_r, K = 2048, 7168, 256, 8
    g = _gen(7168)
    u = _randn((T, d), g, 1.0)
    E = _randn((N_r, d), g, d ** -0.5)
    b = ((torch.rand(N_r, generator=g, device=DEV) * 2 - 1) * 0.01).float()
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    gate = torch.empty(T, K, dtype=torch.float32, device=DEV)
    counts = torch.empty(N_r, dtype=torch.int32, device=DEV)
    ws = _ws(moe.moe_route_workspace_size(T, N_r))
    moe.moe_route(u, E, b, K, idx, gate, counts, ws)
    torch.cuda.synchronize()
    assert _listed_tokens(ws, T, N_r) > 0, "no token reached the float64 tie-break"
    ref = O.route(f64(u), f64(E), b.cpu().numpy(), K)
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy(), ref, K,
                  gate_tol=GATE_TOL["bf16"])


def test_route_grouped_group_choice_moved_by_tie_break():
    """Experts 24 (group 3) and 32 (group 4) differ in one centroid entry and
    carry the same bias, so the 4th and 5th group scores are closer than the
    float32 logit error for many tokens: where the float32 logits order the
    two the wrong way, the float64 tie-break moves the group choice and the
    new group's experts near the (K+1)-th key get float64 keys too.  Every
    token whose float64 keys are clear of other near-ties must match the
    oracle exactly."""
    T, d, N_r, K, G, M = 2048, 7168, 64, 8, 8, 4
    g = _gen(4242)
    u = _randn((T, d), g, 1.0)
    E = _randn((N_r, d), g, d ** -0.5)
    E[32] = E[24]
    E[24, 5] = 0.0
    E[32, 5] = 2.0 ** -19
    b = torch.zeros(N_r, device=DEV)
    b[[0, 8, 16]] = 2.0            # groups 0-2 always kept
    b[[24, 32]] = 1.0              # groups 3 and 4 contend for the last place
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    gate = torch.empty(T, K, dtype=torch.float32, device=DEV)
    counts = torch.empty(N_r, dtype=torch.int32, device=DEV)
    ws = _ws(moe.moe_route_workspace_size(T, N_r))
    ws.fill_(0xFF)                 # float32 logits of unlisted tokens stay NaN
    moe.moe_route_grouped(u, E, b, K, G, M, idx, gate, counts, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    ref = O.route_grouped(f64(u), f64(E), b.cpu().numpy(), K, G, M)
    got = idx.cpu().numpy()
    check_routing(got, gate.cpu().numpy(), counts.cpu().numpy(),
                  grouped_reference(ref, K, G, M), K, gate_tol=GATE_TOL["bf16"])
    # the float32 logits of the listed tokens (white-box: copied to the
    # workspace for the tie-break) put the wrong group first for some tokens
    x32 = ws[:T * N_r * 4].view(torch.float32).view(T, N_r).cpu().numpy()
    listed = ~np.isnan(x32).any(1)
    key = ref["key"]
    f64_g4 = key[:, 32] > key[:, 24]
    moved = listed & ((x32[:, 32] > x32[:, 24]) != f64_g4) & (key[:, 32] != key[:, 24])
    assert moved.sum() > 0, "no token had its group choice moved"
    # exact where the oracle's group choice is not a float32 tie and its
    # selection inside the kept groups has no near-tie
    gs = N_r // G
    gsc = key.reshape(T, G, gs).max(2)
    kept = np.zeros((T, G), bool)
    np.put_along_axis(kept, np.argsort(-gsc, axis=1, kind="stable")[:, :M], True, axis=1)
    masked = np.where(np.repeat(kept, gs, axis=1), key, -np.inf)
    sel_gap, ord_gap = O.topk_margins(masked, ref["idx"])
    strict = (key[:, 32] != key[:, 24]) & (sel_gap >= TIE_GAP) & (ord_gap >= TIE_GAP)
    assert strict[moved].sum() > 0
    bad = strict & np.any(got != ref["idx"], axis=1)
    assert not bad.any(), f"{int(bad.sum())} of {int(strict.sum())} tokens differ " \
        f"({int((bad & moved).sum())} with a moved group choice)"


@pytest.mark.parametrize("grouped", [False, True])
def test_route_duplicate_centroids_exact_ties(grouped):
    """Experts 2j and 2j+1 share a centroid and b = 0: every key is tied, every
    token goes through the float64 tie-break, and ties go to the lower index."""
    T, d, N_r, K = 600, 512, 64, 6
    g = _gen(99)
    u = _randn((T, d), g)
    E = _randn((N_r // 2, d), g, d ** -0.5).repeat_interleave(2, dim=0).contiguous()
    b = torch.zeros(N_r, device=DEV)
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    gate = torch.empty(T, K, dtype=torch.float32, device=DEV)
    counts = torch.empty(N_r, dtype=torch.int32, device=DEV)
    ws = _ws(moe.moe_route_workspace_size(T, N_r))
    if grouped:
        moe.moe_route_grouped(u, E, b, K, 8, 3, idx, gate, counts, ws)
    else:
        moe.moe_route(u, E, b, K, idx, gate, counts, ws)
    torch.cuda.synchronize()
    assert _listed_tokens(ws, T, N_r) == T
    got = idx.cpu().numpy()
    if grouped:
        ref = O.route_grouped(f64(u), f64(E), b.cpu().numpy(), K, 8, 3)
        check_routing(got, gate.cpu().numpy(), counts.cpu().numpy(),
                      grouped_reference(ref, K, 8, 3), K, gate_tol=GATE_TOL["bf16"])
    else:
        ref = O.route(f64(u), f64(E), b.cpu().numpy(), K)
        check_routing(got, gate.cpu().numpy(), counts.cpu().numpy(), ref, K,
                      gate_tol=GATE_TOL["bf16"])
    # K even: both members of each chosen pair are selected, lower index first
    assert (got[:, 0::2] % 2 == 0).all() and (got[:, 1::2] == got[:, 0::2] + 1).all()


def test_route_zero_centroids_gates_are_uniform():
    """E = 0: s = 1/2 everywhere, selection follows b, gates are exactly 1/K."""
    T, d, N_r, K = 100, 256, 64, 4
    u = _randn((T, d), _gen(1))
    E = torch.zeros(N_r, d, dtype=torch.bfloat16, device=DEV)
    b = torch.linspace(-0.01, 0.01, N_r, device=DEV).flip(0).contiguous()
    idx, gate, counts = _route(u, E, b, K)
    assert (idx.cpu() == torch.arange(K, dtype=torch.int32)).all()
    assert (gate.cpu() == 0.25).all()
    assert counts[:K].tolist() == [T] * K and int(counts[K:].sum()) == 0


def test_route_empty_batch():
    N_r = 64
    E = _randn((N_r, 128), _gen(2))
    b = torch.zeros(N_r, device=DEV)
    u = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    idx, gate, counts = _route(u, E, b, 4)
    assert int(counts.abs().sum()) == 0


# ------------------------------------------------------------------ permute

def _rand_idx(T, N_r, K, seed, skew=False):
    rng = np.random.default_rng(seed)
    p = None
    if skew:
        p = 1.0 / np.arange(1, N_r + 1) ** 1.2
        p[N_r // 2: N_r // 2 + 3] = 0           # a few experts never chosen
        p /= p.sum()
    return np.stack([rng.choice(N_r, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,d,N_r,K,dtype", [
    (1000, 256, 64, 6, torch.bfloat16),
    (777, 512, 256, 8, torch.bfloat16),
    (300, 128, 16, 4, torch.float32),
    (513, 256, 32, 2, torch.uint8),           # FP8 rows + tile scales
    (40, 128, 64, 17, torch.bfloat16),        # K > 16 path
    (2000, 128, 1024, 8, torch.bfloat16),     # N_r = 1024, the most the library takes
])
def test_permute_bit_exact(T, d, N_r, K, dtype):
    idx_np = _rand_idx(T, N_r, K, T + K, skew=True)
    g = _gen(T)
    if dtype == torch.uint8:
        u = torch.randint(0, 255, (T, d), generator=g, device=DEV, dtype=torch.uint8)
        u_scale = torch.rand(T, d // 128, generator=g, device=DEV)
        x_scale = torch.empty(T * K, d // 128, device=DEV)
    else:
        u = _randn((T, d), g, 1.0, dtype)
        u_scale = x_scale = None
    idx = torch.from_numpy(idx_np).to(DEV)
    x_perm = torch.empty(T * K, d, dtype=dtype, device=DEV)
    offsets = torch.empty(N_r + 1, dtype=torch.int32, device=DEV)
    perm_src = torch.empty(T * K, dtype=torch.int32, device=DEV)
    inv_row = torch.empty(T, K, dtype=torch.int32, device=DEV)
    ws = _ws(moe.moe_permute_workspace_size(T, N_r))
    moe.moe_permute(u, idx, N_r, x_perm, offsets, perm_src, inv_row, ws, u_scale=u_scale,
                    x_scale=x_scale)
    torch.cuda.synchronize()
    r_off, r_src, r_inv = O.permute_indices(idx_np, N_r)
    np.testing.assert_array_equal(offsets.cpu().numpy(), r_off)
    np.testing.assert_array_equal(perm_src.cpu().numpy(), r_src)
    np.testing.assert_array_equal(inv_row.cpu().numpy(), r_inv)
    src = torch.from_numpy(r_src.astype(np.int64)).to(DEV)
    assert torch.equal(x_perm, u[src])
    if x_scale is not None:
        assert torch.equal(x_scale, u_scale[src])


@pytest.mark.parametrize("T,N_r,K", [(1000, 64, 6), (40, 64, 17), (1, 8, 3)])
def test_permute_index_bit_exact(T, N_r, K):
    """moe_permute_index writes the grouping of moe_permute (offsets,
    perm_src, inv_row) equal to the oracle's, and copies no rows."""
    idx_np = _rand_idx(T, N_r, K, T + 2 * K, skew=True)
    idx = torch.from_numpy(idx_np).to(DEV)
    offsets = torch.empty(N_r + 1, dtype=torch.int32, device=DEV)
    perm_src = torch.empty(T * K, dtype=torch.int32, device=DEV)
    inv_row = torch.empty(T, K, dtype=torch.int32, device=DEV)
    moe.moe_permute_index(idx, N_r, offsets, perm_src, inv_row,
                          _ws(moe.moe_permute_workspace_size(T, N_r)))
    torch.cuda.synchronize()
    r_off, r_src, r_inv = O.permute_indices(idx_np, N_r)
    np.testing.assert_array_equal(offsets.cpu().numpy(), r_off)
    np.testing.assert_array_equal(perm_src.cpu().numpy(), r_src)
    np.testing.assert_array_equal(inv_row.cpu().numpy(), r_inv)


def test_permute_skips_ids_out_of_range():
    """Pairs whose expert id is outside [0, N_r) are left out: inv_row = -1, no
    row copied, and the other pairs keep their stable grouped order."""
    T, d, N_r, K = 300, 128, 32, 4
    idx_np = _rand_idx(T, N_r, K, 5)
    rng = np.random.default_rng(6)
    bad = rng.random((T, K)) < 0.05
    idx_np[bad] = np.where(rng.random(int(bad.sum())) < 0.5, -1, N_r + 3)
    u = _randn((T, d), _gen(3))
    idx = torch.from_numpy(idx_np).to(DEV)
    x_perm = torch.full((T * K, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    offsets = torch.empty(N_r + 1, dtype=torch.int32, device=DEV)
    perm_src = torch.full((T * K,), -5, dtype=torch.int32, device=DEV)
    inv_row = torch.empty(T, K, dtype=torch.int32, device=DEV)
    moe.moe_permute(u, idx, N_r, x_perm, offsets, perm_src, inv_row,
                    _ws(moe.moe_permute_workspace_size(T, N_r)))
    torch.cuda.synchronize()
    # brute force over the valid pairs: grouped by expert, tokens ascending
    pairs = sorted((int(e), t, k) for t in range(T) for k, e in enumerate(idx_np[t])
                   if 0 <= e < N_r)
    want_inv = np.full((T, K), -1, np.int64)
    for r, (e, t, k) in enumerate(pairs):
        want_inv[t, k] = r
    want_off = np.searchsorted([p[0] for p in pairs], np.arange(N_r + 1), side="left")
    np.testing.assert_array_equal(offsets.cpu().numpy(), want_off)
    np.testing.assert_array_equal(inv_row.cpu().numpy(), want_inv)
    n = len(pairs)
    np.testing.assert_array_equal(perm_src.cpu().numpy()[:n], [t for _, t, _ in pairs])
    src = torch.tensor([t for _, t, _ in pairs], device=DEV)
    assert torch.equal(x_perm[:n], u[src])
    assert torch.isnan(x_perm[n:].float()).all()


def test_permute_empty_batch():
    N_r = 32
    offsets = torch.full((N_r + 1,), 5, dtype=torch.int32, device=DEV)
    z = torch.empty(0, 8, dtype=torch.int32, device=DEV)
    u = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    moe.moe_permute(u, z, N_r, torch.empty(0, 128, dtype=torch.bfloat16, device=DEV), offsets,
                    torch.empty(0, dtype=torch.int32, device=DEV), z.clone(), _ws(256))
    torch.cuda.synchronize()
    assert int(offsets.abs().sum()) == 0


# ------------------------------------------------------------------ expert FFN

def _groups(sizes):
    off = np.zeros(len(sizes) + 1, np.int32)
    off[1:] = np.cumsum(sizes)
    return off


def _ffn_case(sizes, d, I, dtype, seed, extra_rows=0):
    g = _gen(seed)
    G = len(sizes)
    off = _groups(sizes)
    rows = int(off[-1]) + extra_rows
    x = _randn((rows, d), g, 1.0, dtype)
    wgu = _randn((G, 2 * I, d), g, d ** -0.5, dtype)
    wdn = _randn((G, d, I), g, I ** -0.5, dtype)
    y = torch.full((rows, d), float("nan"), dtype=dtype, device=DEV)
    dt = moe.MOE_F32 if dtype == torch.float32 else moe.MOE_BF16
    ws = _ws(moe.moe_expert_ffn_workspace_size(dt, rows, I))
    offsets = torch.from_numpy(off).to(DEV)
    moe.moe_expert_ffn(x, offsets, wgu, wdn, y, ws)
    torch.cuda.synchronize()
    ex = LazyExperts(wgu, wdn)
    xs = f64(x)
    ref = np.zeros((int(off[-1]), d))
    for e in range(G):
        a, b_ = int(off[e]), int(off[e + 1])
        if b_ > a:
            ref[a:b_] = O.swiglu_ffn(xs[a:b_], *ex[e])
    got = f64(y)
    return got, ref, int(off[-1])


@pytest.mark.parametrize("sizes,d,I", [
    ([0, 1, 127, 128, 129, 300, 0, 5], 256, 256),   # ragged groups, empty groups
    ([64, 200, 333], 512, 384),                     # I not a multiple of 256
    ([1000, 700, 1300, 60], 1024, 512),             # many tiles per CTA, stage wrap-around
    ([5000], 768, 256),                             # one large group (the shared-expert shape)
    ([64, 200, 333], 384, 256),                     # d not a multiple of 256 (128-column down tiles)
    ([255, 256, 257, 511, 513, 17, 16, 15], 256, 128),  # token tiling around 256-row boundaries
    # tiny, empty and 256-row boundary groups with 256-column weight tiles on both GEMMs
    ([255, 256, 257, 511, 513, 17, 16, 15, 1, 8, 9, 0, 24], 512, 256),
    ([3] * 40 + [700, 0, 129], 1024, 768),            # many small groups, 3 gate/up pair tiles
])
def test_expert_ffn_bf16(sizes, d, I):
    got, ref, n = _ffn_case(sizes, d, I, torch.bfloat16, sum(sizes) + d, extra_rows=3)
    assert_close(got[:n], ref, TOL["bf16"], "y")
    assert np.isnan(got[n:]).all(), "rows outside every group were written"
    assert moe.moe_device_status() == 0


def _max_group_sizes(seed):
    """1024 ragged groups (the most a grouped launch takes): ~40 % empty, the
    rest 1-40 rows, one of 300 rows (two 256-row token tiles)."""
    rng = np.random.default_rng(seed)
    sizes = np.where(rng.random(1024) < 0.4, 0, rng.integers(1, 41, 1024))
    sizes[517] = 300
    return sizes.tolist()


def test_expert_ffn_bf16_max_groups():
    got, ref, n = _ffn_case(_max_group_sizes(1), 256, 128, torch.bfloat16, 1024, extra_rows=3)
    assert_close(got[:n], ref, TOL["bf16"], "y")
    assert np.isnan(got[n:]).all(), "rows outside every group were written"
    assert moe.moe_device_status() == 0


def test_expert_ffn_fp8_max_groups():
    got, ref = _fp8_ffn_case(_max_group_sizes(2), 256, 128, 1025)
    assert_close(got, ref, TOL["e4m3"], "y fp8")


def test_expert_ffn_refuses_more_than_1024_groups():
    """1025 groups: MOE_ERR_UNSUPPORTED from the host checks, nothing launched."""
    d, I, G = 256, 128, 1025
    x = torch.zeros(8, d, dtype=torch.bfloat16, device=DEV)
    wgu = torch.zeros(G, 2 * I, d, dtype=torch.bfloat16, device=DEV)
    wdn = torch.zeros(G, d, I, dtype=torch.bfloat16, device=DEV)
    offsets = torch.zeros(G + 1, dtype=torch.int32, device=DEV)
    y = torch.empty(8, d, dtype=torch.bfloat16, device=DEV)
    ws = _ws(moe.moe_expert_ffn_workspace_size(moe.MOE_BF16, 8, I))
    with pytest.raises(moe.MoeError, match="MOE_ERR_UNSUPPORTED"):
        moe.moe_expert_ffn(x, offsets, wgu, wdn, y, ws)


def test_expert_ffn_clamps_bad_offsets():
    """Offsets that decrease or run past `rows` are clamped on the device: the
    groups become [0, 100), [100, 100), [100, 250), [250, 250) of 250 rows,
    nothing past row 250 of y is written, moe_device_status reports bit 16,
    and the next call with good offsets is clean."""
    d, I, rows = 256, 128, 250
    g = _gen(4242)
    x = _randn((rows, d), g)
    wgu = _randn((4, 2 * I, d), g, d ** -0.5)
    wdn = _randn((4, d, I), g, I ** -0.5)
    y = torch.full((rows + 40, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = _ws(moe.moe_expert_ffn_workspace_size(moe.MOE_BF16, rows, I))
    bad = torch.tensor([0, 100, 50, 300, 260], dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn(x, bad, wgu, wdn, y[:rows], ws)
    assert moe.moe_device_status() == 16
    got = f64(y)
    assert np.isnan(got[rows:]).all(), "rows past the end were written"
    ex = LazyExperts(wgu, wdn)
    xs = f64(x)
    assert_close(got[:100], O.swiglu_ffn(xs[:100], *ex[0]), TOL["bf16"], "group 0")
    assert_close(got[100:rows], O.swiglu_ffn(xs[100:rows], *ex[2]), TOL["bf16"], "group 2")
    good = torch.tensor([0, 100, 100, 250, 250], dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn(x, good, wgu, wdn, y[:rows], ws)
    assert moe.moe_device_status() == 0


@pytest.mark.parametrize("sizes,d,I", [([3, 0, 64, 65, 130], 256, 128), ([200], 128, 256)])
def test_expert_ffn_f32(sizes, d, I):
    got, ref, n = _ffn_case(sizes, d, I, torch.float32, 7 + d)
    assert_close(got[:n], ref, TOL["f32"], "y")


# ------------------------------------------------------------------ combine, bias

@pytest.mark.parametrize("T,d,K,N_s,dtype", [
    (1000, 512, 6, 2, torch.bfloat16), (333, 256, 8, 1, torch.bfloat16),
    (200, 128, 4, 0, torch.float32), (64, 256, 17, 1, torch.bfloat16),
    (77, 7168, 8, 1, torch.bfloat16),     # V3 row: seven 2 KB chunks, a partial token group
    (130, 1536, 16, 3, torch.bfloat16),   # K = 16, ragged last chunk (3072 B rows)
    (50, 2560, 16, 2, torch.float32),     # float32 rows of five chunks
    (41, 1024, 16, 40, torch.bfloat16),   # 57 row slots: 512-byte chunks, four stages
])
def test_combine(T, d, K, N_s, dtype):
    g = _gen(T + K)
    u = _randn((T, d), g, 1.0, dtype)
    ys = _randn((N_s, T, d), g, 0.5, dtype) if N_s else None
    yp = _randn((T * K, d), g, 0.5, dtype)
    perm = torch.randperm(T * K, generator=torch.Generator().manual_seed(T))
    inv = perm.view(T, K).to(torch.int32).to(DEV)
    gate = torch.rand(T, K, generator=g, device=DEV)
    gate = (gate / gate.sum(1, keepdim=True)).contiguous()
    out = torch.empty(T, d, dtype=dtype, device=DEV)
    moe.moe_combine(u, ys, yp, inv, gate, out)
    torch.cuda.synchronize()
    ref = f64(u) + (f64(ys).sum(0) if N_s else 0)
    ref = ref + np.einsum("tk,tkd->td", f64(gate), f64(yp)[inv.long().cpu().numpy()])
    tol = TOL["f32"] if dtype == torch.float32 else 2 ** -8
    assert_close(f64(out), ref, tol, "h'")


def test_combine_skips_rows_left_out():
    """A slot whose grouped row is -1 (an expert id the permute left out)
    contributes nothing."""
    T, d, K = 90, 1024, 8
    g = _gen(5)
    u = _randn((T, d), g)
    yp = _randn((T * K, d), g, 0.5)
    inv = torch.randperm(T * K, generator=torch.Generator().manual_seed(1)).view(T, K)
    inv[::7, 3] = -1
    inv = inv.to(torch.int32).to(DEV)
    gate = torch.rand(T, K, generator=g, device=DEV)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(u, None, yp, inv, gate, out)
    torch.cuda.synchronize()
    iv = inv.long().cpu().numpy()
    w = np.where(iv >= 0, f64(gate), 0.0)
    ref = f64(u) + np.einsum("tk,tkd->td", w, f64(yp)[np.maximum(iv, 0)])
    assert_close(f64(out), ref, 2 ** -8, "h'")


def _bwd_case(T, d, K, N_s, dtype, seed):
    g = _gen(seed)
    N_r = 3 * K
    u = _randn((T, d), g, 1.0, dtype)
    E = _randn((N_r, d), g, d ** -0.5, dtype)
    dh = _randn((T, d), g, 0.1, dtype)
    yp = _randn((T * K, d), g, 0.5, dtype)
    dxp = _randn((T * K, d), g, 0.1, dtype)
    dxs = _randn((N_s, T, d), g, 0.1, dtype) if N_s else None
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(N_r, K, replace=False) for _ in range(T)]).astype(np.int32)
    inv = rng.permutation(T * K).reshape(T, K).astype(np.int32)
    # gates as the router makes them: g = s / sum(s) over the selected experts
    s_sel = B.sigmoid(np.einsum("td,tkd->tk", f64(u), f64(E)[idx]))
    gate = torch.from_numpy(s_sel / s_sel.sum(1, keepdims=True)).float().to(DEV)
    return u, E, dh, yp, dxp, dxs, idx, inv, gate


@pytest.mark.parametrize("T,d,K,N_s,dtype", [
    (77, 7168, 8, 1, torch.bfloat16),     # V3 rows, a partial token group
    (130, 1536, 16, 2, torch.bfloat16),   # K = 16, ragged last chunk
    (45, 2560, 16, 0, torch.float32),
    (333, 256, 6, 3, torch.float32),      # rows shorter than one chunk
    (64, 256, 3, 1, torch.bfloat16),      # small K
    (37, 1536, 16, 20, torch.bfloat16),   # 53 row slots: 512-byte chunks, four stages
])
def test_combine_and_unpermute_backward(T, d, K, N_s, dtype):
    """moe_combine_backward and moe_unpermute_backward against the chain rule
    written out with the oracle's gate backward (selection held fixed)."""
    u, E, dh, yp, dxp, dxs, idx, inv, gate = _bwd_case(T, d, K, N_s, dtype, T + d + K)
    idx_d = torch.from_numpy(idx).to(DEV)
    inv_d = torch.from_numpy(inv).to(DEV)
    dyp = torch.full((T * K, d), float("nan"), dtype=dtype, device=DEV)
    d_gate = torch.empty(T, K, device=DEV)
    d_logit = torch.empty(T, K, device=DEV)
    d_logit_perm = torch.empty(T * K, device=DEV)
    moe.moe_combine_backward(dh, u, E, yp, inv_d, idx_d, gate, dyp, d_gate, d_logit, d_logit_perm)
    du = torch.empty(T, d, dtype=dtype, device=DEV)
    moe.moe_unpermute_backward(dh, dxs, dxp, inv_d, idx_d, d_logit, E, du)
    torch.cuda.synchronize()
    tol = TOL["f32"] if dtype == torch.float32 else TOL["bf16"]
    g64, dh64, ys = f64(gate), f64(dh), f64(yp)
    want_dyp = np.zeros((T * K, d))
    want_dyp[inv] = g64[:, :, None] * dh64[:, None, :]
    assert_close(f64(dyp), want_dyp, tol, "dy_perm")
    want_dg = np.einsum("td,tkd->tk", dh64, ys[inv])
    assert_close(d_gate.double().cpu().numpy(), want_dg, tol, "d_gate")
    s_sel = B.sigmoid(np.einsum("td,tkd->tk", f64(u), f64(E)[idx]))
    want_dl = B.gate_backward(s_sel, want_dg) * s_sel * (1 - s_sel)
    assert_close(d_logit.double().cpu().numpy(), want_dl, tol, "d_logit")
    assert_close(d_logit_perm.double().cpu().numpy()[inv], want_dl, tol, "d_logit_perm")
    dl = d_logit.double().cpu().numpy()
    want_du = dh64 + (f64(dxs).sum(0) if N_s else 0) + f64(dxp)[inv].sum(1) + \
        np.einsum("tk,tkd->td", dl, f64(E)[idx])
    assert_close(f64(du), want_du, tol, "du")
    assert moe.moe_device_status() == 0


def test_combine_wait_that_runs_out_is_reported_and_next_call_is_clean():
    """With the pipeline's wait bound cut to 1 ns, a wait on a stage whose
    copies are still in flight runs out: the kernel stops, returns, and
    moe_device_status reports bit 8 (no fault, no hang).  With the default
    bound restored the same call is clean and correct."""
    T, d, K, N_s = 4096, 7168, 8, 1
    g = _gen(808)
    u = _randn((T, d), g)
    ys = _randn((N_s, T, d), g, 0.5)
    yp = _randn((T * K, d), g, 0.5)
    inv = torch.randperm(T * K, generator=torch.Generator().manual_seed(3)).view(T, K)
    inv = inv.to(torch.int32).to(DEV)
    gate = torch.rand(T, K, generator=g, device=DEV)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    assert moe.moe_device_status() == 0
    try:
        moe.moe_set_pipeline_wait_limit(1)
        moe.moe_combine(u, ys, yp, inv, gate, out)
        assert moe.moe_device_status() == 8
    finally:
        moe.moe_set_pipeline_wait_limit(0)
    moe.moe_combine(u, ys, yp, inv, gate, out)
    assert moe.moe_device_status() == 0
    rows = np.arange(0, T, 97)
    iv = inv.long().cpu().numpy()[rows]
    ref = f64(u)[rows] + f64(ys)[0][rows] + np.einsum("tk,tkd->td", f64(gate)[rows],
                                                      f64(yp)[iv])
    assert_close(f64(out)[rows], ref, 2 ** -8, "h' after the timeout")


def test_backward_leaves_out_slots_with_bad_expert_ids():
    """Slots whose expert id is -1 or N_r (moe_permute gives them inv_row -1)
    are left out of the backward: the selection is the remaining slots, so
    d_gate and d_logit of the left-out slot are 0, no dy_perm row or
    d_logit_perm entry is written, and the gate backward of the oracle runs
    over the valid slots only; no centroid row outside E is read."""
    T, d, K, N_s = 93, 1024, 8, 1
    u, E, dh, yp, dxp, dxs, idx, inv, gate = _bwd_case(T, d, K, N_s, torch.bfloat16, 77)
    N_r = E.shape[0]
    rng = np.random.default_rng(5)
    bad = rng.random((T, K)) < 0.12
    bad[0, :] = False
    bad[1, 2] = True
    idx = idx.copy()
    idx[bad] = np.where(rng.random(int(bad.sum())) < 0.5, -1, N_r)
    inv = inv.copy()
    inv[bad] = -1
    s_all = B.sigmoid(np.einsum("td,tkd->tk", f64(u), f64(E)[np.clip(idx, 0, N_r - 1)]))
    s_all[bad] = 0.0
    g64 = s_all / s_all.sum(1, keepdims=True)
    gate = torch.from_numpy(g64).float().to(DEV)
    idx_d = torch.from_numpy(idx).to(DEV)
    inv_d = torch.from_numpy(inv).to(DEV)
    dyp = torch.full((T * K, d), 3.0, dtype=torch.bfloat16, device=DEV)
    d_gate = torch.full((T, K), 9.0, device=DEV)
    d_logit = torch.full((T, K), 9.0, device=DEV)
    d_logit_perm = torch.full((T * K,), 9.0, device=DEV)
    moe.moe_combine_backward(dh, u, E, yp, inv_d, idx_d, gate, dyp, d_gate, d_logit, d_logit_perm)
    du = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    moe.moe_unpermute_backward(dh, dxs, dxp, inv_d, idx_d, d_logit, E, du)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    tol = TOL["bf16"]
    dh64, ys = f64(dh), f64(yp)
    ok = ~bad
    want_dg = np.where(ok, np.einsum("td,tkd->tk", dh64, ys[np.maximum(inv, 0)]), 0.0)
    want_dl = np.zeros((T, K))
    for t in range(T):
        v = ok[t]
        ds = B.gate_backward(s_all[t:t + 1, v], want_dg[t:t + 1, v])[0]
        want_dl[t, v] = ds * s_all[t, v] * (1 - s_all[t, v])
    got_dg = d_gate.double().cpu().numpy()
    got_dl = d_logit.double().cpu().numpy()
    assert np.all(got_dg[bad] == 0) and np.all(got_dl[bad] == 0)
    assert_close(got_dg, want_dg, tol, "d_gate")
    assert_close(got_dl, want_dl, tol, "d_logit")
    written = np.zeros(T * K, bool)
    written[inv[ok]] = True
    dlp = d_logit_perm.double().cpu().numpy()
    assert np.all(dlp[~written] == 9.0)                     # left-out rows untouched
    assert_close(dlp[inv[ok]], want_dl[ok], tol, "d_logit_perm")
    got_dyp = f64(dyp)
    assert np.all(got_dyp[~written] == 3.0)
    want_dyp = g64[:, :, None] * dh64[:, None, :]
    assert_close(got_dyp[inv[ok]], want_dyp[ok], tol, "dy_perm")
    want_du = dh64 + f64(dxs).sum(0)
    for t in range(T):
        for k in range(K):
            if ok[t, k]:
                want_du[t] += f64(dxp)[inv[t, k]] + got_dl[t, k] * f64(E)[idx[t, k]]
    assert_close(f64(du), want_du, tol, "du")


def test_bias_update_bit_exact():
    N_r, T, K = 256, 8192, 8            # mean load 256
    rng = np.random.default_rng(3)
    counts = rng.integers(200, 313, N_r).astype(np.int32)
    counts[:10] = 256                   # equal to the mean: unchanged
    b = rng.uniform(-0.05, 0.05, N_r).astype(np.float32)
    bd = torch.from_numpy(b).to(DEV)
    moe.moe_bias_update(bd, torch.from_numpy(counts).to(DEV), T, K, 0.001)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bd.cpu().numpy(), O.bias_update(b, counts, T, K))


# ------------------------------------------------------------------ FP8 quantisers

def _e4m3_values(q_u8):
    return q_u8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_quantize_1x128_bit_exact():
    g = _gen(5)
    x = _randn((300, 7 * 128), g, 1.0)
    mask = torch.rand(300, 7 * 128, generator=g, device=DEV) < 0.001
    x = torch.where(mask, x * 50, x).to(torch.bfloat16)
    x[7, 128:256] = 0
    q = torch.empty(300, 896, dtype=torch.uint8, device=DEV)
    s = torch.empty(300, 7, device=DEV)
    moe.moe_quantize_1x128(x, q, s)
    torch.cuda.synchronize()
    rq, rs = O.quant_1x128(f64(x).astype(np.float32))
    np.testing.assert_array_equal(s.cpu().numpy(), rs)
    np.testing.assert_array_equal(_e4m3_values(q), rq)


def test_quantize_1x128_every_bf16_value_bit_exact():
    """Every finite bf16 value x with |x| below the tile's amax, in tiles of 127
    such values plus one amax (several amax values, so the quotients x/scale
    land everywhere on the E4M3 grid, its rounding midpoints included): codes
    and scales equal the oracle's IEEE-division quantisation bit for bit."""
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    allv = bits.view(torch.bfloat16).float()
    finite = allv[torch.isfinite(allv)]
    rows = []
    for amax in (1.0, 0.7, 3.140625, 0.0009765625, 250.0):
        v = finite[finite.abs() < amax]
        v = v[torch.randperm(v.numel(), generator=torch.Generator().manual_seed(7))]
        pad = (-v.numel()) % 127
        v = torch.cat([v, torch.zeros(pad)]).view(-1, 127)
        rows.append(torch.cat([v, torch.full((v.shape[0], 1), amax)], dim=1))
    x = torch.cat(rows).to(torch.bfloat16)                     # [tiles, 128]
    n = x.shape[0] // 7 * 7
    x = x[:n].reshape(n // 7, 7 * 128).contiguous().to(DEV)    # 7 tiles per row
    q = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
    s = torch.empty(x.shape[0], 7, device=DEV)
    moe.moe_quantize_1x128(x, q, s)
    torch.cuda.synchronize()
    rq, rs = O.quant_1x128(f64(x).astype(np.float32))
    np.testing.assert_array_equal(s.cpu().numpy(), rs)
    np.testing.assert_array_equal(_e4m3_values(q), rq)


def test_quantize_128x128_bit_exact():
    g = _gen(6)
    w = _randn((3, 256, 384), g, 0.02)
    q = torch.empty(3, 256, 384, dtype=torch.uint8, device=DEV)
    s = torch.empty(3, 2, 3, device=DEV)
    moe.moe_quantize_128x128(w, q, s)
    torch.cuda.synchronize()
    for e in range(3):
        rq, rs = O.quant_128x128(f64(w[e]).astype(np.float32))
        np.testing.assert_array_equal(s[e].cpu().numpy(), rs)
        np.testing.assert_array_equal(_e4m3_values(q[e]), rq)


# ------------------------------------------------------------------ FP8 expert FFN

def _fp8_ffn_case(sizes, d, I, seed, outliers=False):
    g = _gen(seed)
    G = len(sizes)
    off = _groups(sizes)
    rows = int(off[-1])
    x = _randn((rows, d), g, 1.0)
    if outliers:
        mask = torch.rand(rows, d, generator=g, device=DEV) < 0.001
        x = torch.where(mask, x.float() * 50, x.float()).to(torch.bfloat16)
    wgu = _randn((G, 2 * I, d), g, d ** -0.5)
    wdn = _randn((G, d, I), g, I ** -0.5)
    xq = torch.empty(rows, d, dtype=torch.uint8, device=DEV)
    xs = torch.empty(rows, d // 128, device=DEV)
    moe.moe_quantize_1x128(x, xq, xs)
    qgu = torch.empty(G, 2 * I, d, dtype=torch.uint8, device=DEV)
    sgu = torch.empty(G, 2 * I // 128, d // 128, device=DEV)
    qdn = torch.empty(G, d, I, dtype=torch.uint8, device=DEV)
    sdn = torch.empty(G, d // 128, I // 128, device=DEV)
    moe.moe_quantize_128x128(wgu, qgu, sgu)
    moe.moe_quantize_128x128(wdn, qdn, sdn)
    y = torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = _ws(moe.moe_expert_ffn_workspace_size(moe.MOE_E4M3, rows, I))
    offsets = torch.from_numpy(off).to(DEV)
    moe.moe_expert_ffn(xq, offsets, qgu, qdn, y, ws, x_scale=xs, w_scale_gate_up=sgu,
                       w_scale_down=sdn)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    # the oracle quantises from the bf16 originals itself
    ex = LazyExperts(wgu, wdn)
    xs64 = f64(x)
    ref = np.zeros((rows, d))
    for e in range(G):
        a, b_ = int(off[e]), int(off[e + 1])
        if b_ > a:
            wg_, wu_, wd_ = ex[e]
            Wq = O.quantise_expert(wg_.astype(np.float32), wu_.astype(np.float32),
                                   wd_.astype(np.float32))
            ref[a:b_] = O.fp8_swiglu_ffn(xs64[a:b_].astype(np.float32), Wq)
    return f64(y), ref


@pytest.mark.parametrize("sizes,d,I,outliers", [
    ([0, 1, 127, 128, 129, 300, 0, 5], 256, 256, False),
    ([64, 200, 333], 512, 384, True),
    ([1000, 700, 1300, 60], 1024, 512, False),
])
def test_expert_ffn_fp8(sizes, d, I, outliers):
    got, ref = _fp8_ffn_case(sizes, d, I, sum(sizes) + 3 * d, outliers)
    assert_close(got, ref, TOL["e4m3"], "y fp8")


def test_expert_gate_up_fp8_codes_close():
    """The FP8 gate/up half alone: its E4M3 codes and 1x128 scales against the
    oracle's h quantisation (ties of the float32 h may round differently, so
    codes agree for nearly all elements and scales closely)."""
    g = _gen(77)
    rows, d, I = 384, 512, 256
    x = _randn((rows, d), g, 1.0)
    wgu = _randn((1, 2 * I, d), g, d ** -0.5)
    xq = torch.empty(rows, d, dtype=torch.uint8, device=DEV)
    xs = torch.empty(rows, d // 128, device=DEV)
    moe.moe_quantize_1x128(x, xq, xs)
    qgu = torch.empty(1, 2 * I, d, dtype=torch.uint8, device=DEV)
    sgu = torch.empty(1, 2 * I // 128, d // 128, device=DEV)
    moe.moe_quantize_128x128(wgu, qgu, sgu)
    h = torch.empty(rows, I, dtype=torch.uint8, device=DEV)
    hs = torch.empty(rows, I // 128, device=DEV)
    offsets = torch.tensor([0, rows], dtype=torch.int32, device=DEV)
    moe.moe_expert_gate_up(xq, offsets, qgu, h, x_scale=xs, w_scale_gate_up=sgu, h_scale=hs)
    torch.cuda.synchronize()
    gu = f64(wgu[0]).astype(np.float32)
    qx, sx = O.quant_1x128(f64(x).astype(np.float32))
    qg, sg = O.quant_128x128(gu[:I])
    qu, su = O.quant_128x128(gu[I:])
    hg = O.fp8_promoted_gemm(qx, sx, qg, sg)
    hu = O.fp8_promoted_gemm(qx, sx, qu, su)
    href = (O.silu(hg) * hu).astype(np.float32)
    rq, rs = O.quant_1x128(href)
    np.testing.assert_allclose(hs.cpu().numpy(), rs, rtol=1e-5)
    codes_equal = (_e4m3_values(h) == rq).mean()
    assert codes_equal > 0.999, codes_equal


@pytest.mark.parametrize("sizes,T,N_s,d,I", [
    ([0, 1, 127, 300, 5, 256], 700, 1, 512, 256),   # ragged routed groups + one shared expert
    ([64, 200, 333], 1000, 2, 256, 384),            # two shared experts, I not a multiple of 256
    ([0, 0, 0], 257, 1, 256, 128),                  # no routed rows: the shared experts alone
])
def test_expert_ffn_with_shared_groups(sizes, T, N_s, d, I):
    """The shared experts as extra groups of the routed launches: routed rows
    as moe_expert_ffn, shared expert j's rows at rows + j*T, equal to the
    oracle's FFN of u; nothing past the last row is written."""
    g = _gen(T + d + N_s)
    G = len(sizes)
    off = _groups(sizes)
    rows = int(off[-1])
    x = _randn((max(rows, 1), d), g)[:rows] if rows else torch.empty(0, d, dtype=torch.bfloat16,
                                                                          device=DEV)
    u = _randn((T, d), g)
    wgu = _randn((G, 2 * I, d), g, d ** -0.5)
    wdn = _randn((G, d, I), g, I ** -0.5)
    wsgu = _randn((N_s, 2 * I, d), g, d ** -0.5)
    wsdn = _randn((N_s, d, I), g, I ** -0.5)
    h = torch.empty(rows + N_s * T, I, dtype=torch.bfloat16, device=DEV)
    y = torch.full((rows + N_s * T + 5, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    offsets = torch.from_numpy(off).to(DEV)
    moe.moe_expert_gate_up_shared(x if rows else u[:0], offsets, wgu, u, wsgu, h)
    moe.moe_expert_down_shared(h, offsets, wdn, wsdn, rows, T, y[:rows + N_s * T])
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    got = f64(y)
    assert np.isnan(got[rows + N_s * T:]).all()
    ex, exs = LazyExperts(wgu, wdn), LazyExperts(wsgu, wsdn)
    if rows:
        xs = f64(x)
        ref = np.zeros((rows, d))
        for e in range(G):
            a, b_ = int(off[e]), int(off[e + 1])
            if b_ > a:
                ref[a:b_] = O.swiglu_ffn(xs[a:b_], *ex[e])
        assert_close(got[:rows], ref, TOL["bf16"], "routed rows")
    us = f64(u)
    for j in range(N_s):
        assert_close(got[rows + j * T: rows + (j + 1) * T], O.swiglu_ffn(us, *exs[j]),
                     TOL["bf16"], f"shared expert {j}")


# B, the bound on the float32 key error behind the router's tie-break (refine
# gap 2B, near distance 3B; include/moe.h, moe_route).
KEY_ERROR_BOUND = 2e-5


@pytest.mark.parametrize("config,step", [("v3_bf16", None), ("v3_zipf_bf16", 0),
                                         ("v3_zipf_bf16", 1)])
def test_router_float32_key_error_within_bound(config, step):
    """With every token re-routed (refine gap 1e30, near 0) the workspace holds
    the fused router's float32 logits for every token.  At the V3 width
    (d 7168, 256 experts, 8192 tokens) on the V3 recipe and on the skewed
    recipe (centroid norms up to 5, logits up to ~22) every key's float32
    error against the float64 affinity stays below B; the routing of the
    fully re-routed batch equals the oracle's."""
    from mixture_experts_layer_60_b200.configs import CONFIGS
    from mixture_experts_layer_60_b200.synth import make_layer_inputs, step_u
    cfg = CONFIGS[config]
    w = make_layer_inputs(cfg, DEV)
    u = w["u"] if step is None else step_u(cfg, step, DEV)
    E, b = w["E"], w["b"]
    T, N_r, K = u.shape[0], E.shape[0], cfg.K
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    gate = torch.empty(T, K, dtype=torch.float32, device=DEV)
    counts = torch.empty(N_r, dtype=torch.int32, device=DEV)
    ws = _ws(moe.moe_route_workspace_size(T, N_r))
    moe.moe_set_router_tie_break(1e30, 0.0)
    try:
        moe.moe_route(u, E, b, K, idx, gate, counts, ws)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_router_tie_break()
    assert moe.moe_device_status() == 0
    assert _listed_tokens(ws, T, N_r) == T
    x32 = ws[:T * N_r * 4].view(torch.float32).view(T, N_r)
    x64 = u.double() @ E.double().T
    s32 = 1.0 / (1.0 + torch.exp(-x32))
    s64 = 1.0 / (1.0 + torch.exp(-x64))
    err = (s32.double() - s64).abs().max().item()
    assert err < KEY_ERROR_BOUND, f"float32 key error {err:.3e} over the bound"
    ref = O.route(f64(u), f64(E), b.cpu().numpy(), K)
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy(), ref, K,
                  gate_tol=GATE_TOL["bf16"])
