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
