"""Host-side accounting of bench.py (no GPU): the layer roofline, the
per-phase algorithmic work and fractions, the launch count per step, the
measured-traffic lookup and the CPU-baseline descriptors.  The figures are
recomputed here from the configuration by hand."""
import math

import bench
from mixture_experts_layer_60_b200.configs import CONFIGS

FALLBACK = {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def test_layer_roofline_v3_bf16():
    cfg = CONFIGS["v3_bf16"]
    tps, flops, nbytes = bench.roofline_layer(cfg, FALLBACK)
    T, d, N_r, K, N_s, I = 8192, 7168, 256, 8, 1, 2048
    assert flops == 2 * T * d * N_r + (K + N_s) * T * 6 * d * I        # 6.524 TFLOP
    assert nbytes == (N_r + N_s) * 3 * I * d * 2 + N_r * d * 2 + 2 * T * d * 2
    t = max(flops / 1590e12, nbytes / 6650e9)
    assert math.isclose(tps, T / t, rel_tol=1e-12)
    assert 1.9e6 < tps < 2.1e6


def test_layer_roofline_fp8_uses_twice_the_tensor_peak():
    cfg = CONFIGS["v3_fp8"]
    tps, flops, nbytes = bench.roofline_layer(cfg, FALLBACK)
    t = max(flops / (2 * 1590e12), nbytes / 6650e9)
    assert math.isclose(tps, cfg.T / t, rel_tol=1e-12)


def test_phase_rooflines_fractions_and_bounds():
    cfg = CONFIGS["v3_bf16"]
    ms = {"route": 0.1, "permute": 0.2, "gate_up": 4.0, "down": 2.0, "combine": 0.3}
    ph = bench.phase_rooflines(cfg, FALLBACK, ms, merged_shared=True)
    assert set(ph) == set(ms)
    T, d, K, N_s, I, N_r = 8192, 7168, 8, 1, 2048, 256
    R = T * K
    # HBM phases: bytes as stated, GB/s from the time, fraction of the copy peak
    assert ph["permute"]["bytes_per_launch"] == T * d * 2 + R * d * 2 + R * 12
    assert ph["combine"]["bytes_per_launch"] == T * d * 2 * (2 + N_s + K) + R * 8
    for name in ("route", "permute", "combine"):
        e = ph[name]
        assert e["bound"] == "hbm" and e["unit"] == "GB/s"
        assert math.isclose(e["achieved"], e["bytes_per_launch"] / (ms[name] * 1e-3) / 1e9)
        assert math.isclose(e["frac"], e["achieved"] / 6650.0)
    # GEMM phases: routed + shared rows; at V3 density both sit tensor-bound
    rows = R + N_s * T
    assert ph["gate_up"]["flops_per_launch"] == 2.0 * rows * d * 2 * I
    assert ph["down"]["flops_per_launch"] == 2.0 * rows * I * d
    for name in ("gate_up", "down"):
        e = ph[name]
        assert e["bound"] == "tensor" and e["unit"] == "TFLOP/s"
        assert math.isclose(e["achieved"], e["flops_per_launch"] / (ms[name] * 1e-3) / 1e12)
        assert math.isclose(e["frac"], e["achieved"] / 1590.0)
    # weights of 257 groups once, rows in and out
    assert ph["gate_up"]["bytes_per_launch"] == (N_r + N_s) * 2 * I * d * 2 + rows * (d + I) * 2


def test_launches_per_step_match_the_launch_list():
    # fused router + tie-break, hist/scan/rank/scatter, gate/up + down (shared
    # experts merged), combine, bias update: the 10 kernels per step of the
    # V3 launch list
    assert bench.gpu_launches_per_step(CONFIGS["v3_bf16"], True) == 10
    # FP8: + the activation quantiser, shared expert as two more launches
    assert bench.gpu_launches_per_step(CONFIGS["v3_fp8"], False) == 13
    # f32: unfused router (logits, top-K, tie-break), shared experts separate
    c = CONFIGS["tiny_f32"]
    assert bench.gpu_launches_per_step(c, False) == 3 + 4 + 2 + 2 * c.N_s + 1 + 1


def test_measured_traffic_only_for_the_captured_sources():
    cfg = CONFIGS["v3_bf16"]
    m = bench.MEASURED_GATE_UP_TRAFFIC["v3_bf16"]
    want = m["bytes"] if bench.sources_sha(cfg.dtype) == m["sha"] else None
    assert bench.measured_traffic(cfg) == want
    assert bench.measured_traffic(CONFIGS["v3_fp8"]) is None


def test_cpu_baseline_descriptors():
    assert bench.cpu_cores() >= 1
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()
