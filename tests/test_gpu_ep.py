"""Expert parallelism, W ranks emulated on one GPU: each rank keeps N_r/W
experts; its rows are dispatched straight into the experts' ranks' buffers
and the outputs returned to their grouped positions (the exact indexing of
the multi-GPU path).  The result of every rank must equal the single-device
layer on the same tokens bit for bit, and every row must arrive once."""
import pytest
import torch

from mixture_experts_layer_60_b200 import moe_device_status
from mixture_experts_layer_60_b200.configs import LayerConfig
from mixture_experts_layer_60_b200.layer import MoELayer
from mixture_experts_layer_60_b200.parallel_ep import EPGroupEmulated
from mixture_experts_layer_60_b200.synth import make_layer_inputs, step_u
from oracle import moe_oracle as O
from tests.harness import GATE_TOL, TOL, LazyExperts, assert_close, check_routing, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,dtype,N_r,T", [(2, "bf16", 16, 256), (4, "bf16", 16, 200),
                                            (8, "bf16", 32, 96), (4, "f32", 16, 64)])
def test_ep_emulated_equals_single_device(W, dtype, N_r, T):
    cfg = LayerConfig(f"ep_{dtype}", T=T, d=512 if dtype == "bf16" else 256, N_r=N_r, K=4,
                      N_s=1, I=256 if dtype == "bf16" else 128, dtype=dtype, seed=31,
                      bias="uniform")
    w = make_layer_inputs(cfg, "cuda")
    us = [step_u(cfg, s, "cuda") for s in range(W)]
    us[1] = us[1][: T - 17].contiguous()          # ranks may hold different token counts
    grp = EPGroupEmulated(cfg, w, W, T_max=T)
    hs = grp.forward(us)
    torch.cuda.synchronize()
    assert moe_device_status() == 0
    total = sum(int(r.recv_offsets[-1]) for r in grp.ranks)
    assert total == sum(u.shape[0] for u in us) * cfg.K          # every row arrived once
    for s, u in enumerate(us):
        ref = MoELayer(cfg, w, T_max=u.shape[0]).forward(u)
        torch.cuda.synchronize()
        assert torch.equal(hs[s], ref), f"rank {s}"
    # and against the oracle directly: each rank's routing and h'
    routed = LazyExperts(w["W_gate_up"], w["W_down"])
    shared = LazyExperts(w["Ws_gate_up"], w["Ws_down"])
    for s, u in enumerate(us):
        rk, T_s = grp.ranks[s], u.shape[0]
        ref = O.route(f64(u), f64(w["E"]), w["b"].cpu().numpy(), cfg.K)
        _, idx, gate = check_routing(rk.topk_idx[:T_s].cpu().numpy(),
                                     rk.topk_gate[:T_s].cpu().numpy(), rk.counts.cpu().numpy(),
                                     ref, cfg.K, gate_tol=GATE_TOL[dtype])
        want = O.layer_forward(f64(u), idx, gate, routed, shared)
        assert_close(f64(hs[s]), want, TOL[dtype], f"rank {s} h' against the oracle")


def test_ep_emulated_v3_width_eight_ranks():
    """Eight emulated ranks at the V3 shape (d 7168, 256 routed experts, 32 per
    rank, K 8, I 2048), 512 tokens per rank (one rank 495): every rank's h'
    equals the single-device layer bit for bit, every row arrives once, and
    32 sampled tokens per rank match the oracle."""
    import numpy as np
    from mixture_experts_layer_60_b200.configs import CONFIGS
    from tests.harness import oracle_layer_rows
    W, T = 8, 512
    cfg = CONFIGS["v3_bf16"].with_T(T)
    w = make_layer_inputs(cfg, "cuda")
    us = [step_u(cfg, s, "cuda") for s in range(W)]
    us[1] = us[1][: T - 17].contiguous()
    grp = EPGroupEmulated(cfg, w, W, T_max=T)
    hs = grp.forward(us)
    torch.cuda.synchronize()
    assert moe_device_status() == 0
    total = sum(int(r.recv_offsets[-1]) for r in grp.ranks)
    assert total == sum(u.shape[0] for u in us) * cfg.K
    single = MoELayer(cfg, w, T_max=T)
    E = f64(w["E"])
    for s, u in enumerate(us):
        ref = single.forward(u)
        torch.cuda.synchronize()
        assert torch.equal(hs[s], ref), f"rank {s}"
        rk, T_s = grp.ranks[s], u.shape[0]
        r = O.route(f64(u), E, w["b"].cpu().numpy(), cfg.K)
        _, idx, gate = check_routing(rk.topk_idx[:T_s].cpu().numpy(),
                                     rk.topk_gate[:T_s].cpu().numpy(), rk.counts.cpu().numpy(),
                                     r, cfg.K, gate_tol=GATE_TOL["bf16"])
        rows = np.sort(np.random.default_rng(s).choice(T_s, 32, replace=False))
        want = oracle_layer_rows(dict(w, u=u), rows, idx[rows], gate[rows])
        assert_close(f64(hs[s])[rows], want, TOL["bf16"], f"rank {s} h' against the oracle")
