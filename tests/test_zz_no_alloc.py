"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory (a host framework that owns every allocation, or a loop that
must not allocate once started), so cannot pass a workspace.  Its scratch is
a static array inside the library.

Checked through the C ABI against moe_permute with a caller workspace, on two
calls in a row (the second smaller than the first, so it runs on scratch
left over from the first).  Index outputs and row copies must match bit for
bit, the same bar as the other permutation tests.  This file is collected
last; it must pass alone in a fresh process and after the other tests."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_60_b200 as moe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(T, d, N_r, K, dtype, seed):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, N_r + 1) ** 1.1
    p /= p.sum()
    idx = np.stack([rng.choice(N_r, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    if dtype == torch.uint8:
        u = torch.randint(0, 255, (T, d), generator=g, device=DEV, dtype=torch.uint8)
        us = torch.rand(T, d // 128, generator=g, device=DEV)
    else:
        u = torch.randn(T, d, generator=g, device=DEV).to(dtype)
        us = None
    return torch.from_numpy(idx).to(DEV), u, us


def _outputs(T, d, N_r, K, dtype, with_scale):
    x = torch.full((T * K, d), 7, dtype=dtype, device=DEV)
    xs = torch.full((T * K, d // 128), -1.0, device=DEV) if with_scale else None
    off = torch.full((N_r + 1,), -1, dtype=torch.int32, device=DEV)
    src = torch.full((T * K,), -1, dtype=torch.int32, device=DEV)
    inv = torch.full((T, K), -1, dtype=torch.int32, device=DEV)
    return x, xs, off, src, inv


def test_noalloc_permute_matches_workspace_permute_on_two_calls():
    cases = [(3000, 512, 256, 8, torch.bfloat16, 11),   # first call: more chunks of scratch
             (700, 256, 64, 6, torch.uint8, 12)]        # second call: fewer, FP8 rows + scales
    for T, d, N_r, K, dtype, seed in cases:
        idx, u, us = _case(T, d, N_r, K, dtype, seed)
        ref = _outputs(T, d, N_r, K, dtype, us is not None)
        ws = torch.empty(max(moe.moe_permute_workspace_size(T, N_r), 256), dtype=torch.uint8,
                         device=DEV)
        moe.moe_permute(u, idx, N_r, ref[0], ref[2], ref[3], ref[4], ws, u_scale=us,
                        x_scale=ref[1])
        got = _outputs(T, d, N_r, K, dtype, us is not None)
        moe.moe_permute_noalloc(u, idx, N_r, got[0], got[2], got[3], got[4], u_scale=us,
                                x_scale=got[1])
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            if a is not None:
                assert torch.equal(a, b)
        assert int(got[2][-1]) == T * K


def test_noalloc_permute_rejects_sizes_beyond_its_static_scratch():
    N_r, K, d = 256, 8, 128
    T = 131072 + 256            # 513 chunks of 256 tokens: 2 * 513 KiB of scratch > 1 MiB
    u = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros(T, K, dtype=torch.int32, device=DEV)
    x, _, off, src, inv = (torch.empty(1, d, dtype=torch.bfloat16, device=DEV), None,
                           torch.empty(N_r + 1, dtype=torch.int32, device=DEV),
                           torch.empty(1, dtype=torch.int32, device=DEV),
                           torch.empty(1, K, dtype=torch.int32, device=DEV))
    with pytest.raises(moe.MoeError, match="static array"):
        moe.moe_permute_noalloc(u, idx, N_r, x, off, src, inv)
