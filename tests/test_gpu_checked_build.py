"""The bounds-checked build (libmoe_checked.so, -DMOE_CHECK_BOUNDS): every
internal index is tested before its access and a failure sets bit 32 of the
device error word instead of trapping.  A child process loads that build
(MOE_LIBRARY) and runs parity tests of every stage of the layer, its
backward and expert parallelism on small ragged shapes, each compared in
full with the oracle; no check may fire."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "mixture_experts_layer_60_b200", "libmoe_checked.so")

CHILD = r"""
import os, sys, torch
sys.path.insert(0, os.getcwd())
import mixture_experts_layer_60_b200 as moe
assert moe.LIB_PATH.endswith("libmoe_checked.so"), moe.LIB_PATH
from tests import test_gpu_kernels as TK, test_gpu_layer as TL, test_gpu_backward as TB
from tests import test_gpu_ep as TE
TK.test_route_matches_oracle(1000, 512, 64, 6, torch.bfloat16)
TK.test_route_grouped_matches_oracle(333, 256, 64, 6, 4, 2)
TK.test_permute_bit_exact(1000, 256, 64, 6, torch.bfloat16)
TK.test_permute_bit_exact(513, 256, 32, 2, torch.uint8)
TK.test_expert_ffn_bf16([255, 256, 257, 511, 513, 17, 16, 15, 1, 8, 9, 0, 24], 512, 256)
TK.test_expert_ffn_bf16([64, 200, 333], 384, 256)
TK.test_expert_ffn_with_shared_groups([0, 1, 127, 300, 5, 256], 700, 1, 512, 256)
TK.test_expert_ffn_fp8([64, 200, 333], 512, 384, True)
TK.test_combine(333, 256, 8, 1, torch.bfloat16)
TL.test_layer_tiny_f32()
TL.test_layer_small_bf16()
TL.test_layer_fp8_small_full()
TB.test_layer_backward_small_full()
TE.test_ep_emulated_equals_single_device(2, "bf16", 16, 256)
torch.cuda.synchronize()
st = moe.moe_device_status()
assert st == 0, f"device error word {st}"
print("checked build ok")
"""


def test_checked_build_runs_every_stage_without_a_bounds_failure():
    assert os.path.exists(CHECKED), "build it with `python -m mixture_experts_layer_60_b200.build --check-bounds`"
    env = dict(os.environ, MOE_LIBRARY=CHECKED)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "checked build ok" in r.stdout
