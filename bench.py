"""Throughput of the DeepSeekMoE layer step on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3_bf16] [--impl ours|reference]

A step is one pass of the whole layer over one batch of synthetic tokens:
route, permute, routed and shared SwiGLU expert FFNs, combine with the
residual, and the per-step bias update (for N > 1 after an all-reduce of the
per-expert load).  Inputs are resident in HBM before the timed region; the
22.6 GB of V3-shaped expert weights stream through HBM every step (far larger
than the 126 MB L2), so no flush is needed between steps.  Timing is CUDA
events on the launching stream, bracketed by a barrier and a device
synchronize, max over ranks.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the C++ one, oracle/moe_ref.cpp) on
the host cores over a bounded token sample per step; with the cpu_baseline
leg it is the only use of oracle/ here.  Expert weights the sample touches
are staged in host memory before the oracle's timer starts.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_60_b200.configs import CONFIGS  # noqa: E402

METRIC = "MoE-layer tokens/sec on 1 B200 + % of roofline (TFLOP/s, HBM GB/s)"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16": j["bf16_tflops"],
                "bf16_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def measure_fp8_peak(dev):
    """Dense E4M3 tensor throughput of this GPU: an 8192^3 torch._scaled_mm
    (unit scales, bf16 out), best of 10 after 3 warm-ups (TFLOP/s)."""
    n = 8192
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev)
    for _ in range(3):
        torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best / 1e3) / 1e12


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "enforced.power.limit")

    def __init__(self, device_index):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        sm, mx, pw, lim, reasons = [], [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2].split()[0]))
                mx.append(float(parts[3].split()[0]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[4].split()[0]))
            except ValueError:
                pass
            try:
                lim.append(float(parts[10].split()[0]))
            except (ValueError, IndexError):
                pass
            for n, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(pw) if pw else None,
                "power_limit_w": max(lim) if lim else None}


# ---------------------------------------------------------------- helpers

def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


# DRAM bytes (read + write) of one routed gate/up launch from an ncu capture
# of a scaled-down case (32 experts, ~256 tokens each) times the units
# processed (weights and rows both scale x8 to the 256-expert launch), with
# the SHA-256 prefix of the kernel sources the capture ran.  The figure is
# reported only while those sources are unchanged; otherwise traffic is null.
KERNEL_SOURCES = {"bf16": ["mixture_experts_layer_60_b200/csrc/gemm_ws.cu",
                           "mixture_experts_layer_60_b200/csrc/sm100.cuh"],
                  "e4m3": ["mixture_experts_layer_60_b200/csrc/gemm_fp8.cu",
                           "mixture_experts_layer_60_b200/csrc/sm100.cuh"]}
# v3_bf16: 2,171,725,824 B read + written by the gate/up launch of 32 experts x
# 256 tokens + the shared expert over 1024 tokens (2,107,637,760 algorithmic
# bytes), scaled by the algorithmic bytes of the 256-expert launch.
MEASURED_GATE_UP_TRAFFIC = {   # workload -> {"bytes": B, "sha": hex prefix}
    "v3_bf16": {"bytes": 16950266033, "sha": "ddfa323d72a58bd3"},
}


def sources_sha(dtype):
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(dtype, []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(cfg):
    m = MEASURED_GATE_UP_TRAFFIC.get(cfg.name)
    if m and m["sha"] == sources_sha(cfg.dtype):
        return m["bytes"]
    return None


def gpu_launches_per_step(cfg, merged_shared):
    # route: the fused router + the float64 tie-break (bf16, N_r <= 256), else
    # logits GEMM + top-K + tie-break; permute: histogram, scan, rank,
    # scatter; expert FFNs: gate/up + down (bf16: the shared experts are
    # extra groups of the same two launches; else 2 more per shared expert);
    # combine: 1; bias update: 1; FP8: + activation quantiser
    fused_router = cfg.dtype != "f32" and cfg.N_r % 32 == 0 and cfg.N_r <= 256 and cfg.K <= 16
    n = (2 if fused_router else 3) + 4 + 2 + (0 if merged_shared else 2 * cfg.N_s) + 1 + 1
    if cfg.dtype == "e4m3":
        n += 1
    return n


def roofline_layer(cfg, p):
    flops = cfg.flops()
    tensor_peak = p["bf16"] * (2 if cfg.dtype == "e4m3" else 1) * 1e12
    bytes_ = cfg.weight_bytes() + cfg.N_r * cfg.d * 2 + 2 * cfg.T * cfg.d * 2
    t = max(flops / tensor_peak, bytes_ / (p["hbm_gbs"] * 1e9))
    return cfg.T / t, flops, bytes_


PHASES = ("route", "permute", "gate_up", "down", "shared", "combine")


def phase_rooflines(cfg, p, phase_ms, merged_shared=False):
    """Per phase of the step: algorithmic FLOPs or HBM bytes per launch (one
    step), achieved rate from the phase's CUDA-event duration, and the
    fraction of the measured peak (burst, and for tensor-bound phases also
    the sustained, power-capped figure).  merged_shared: the gate/up and
    down launches also run the N_s shared experts (T rows each)."""
    T, d, N_r, K, N_s, I = cfg.T, cfg.d, cfg.N_r, cfg.K, cfg.N_s, cfg.I
    R = T * K
    Rg = R + (N_s * T if merged_shared else 0)          # rows of the grouped launches
    Gw = N_r + (N_s if merged_shared else 0)            # weight groups they stream
    fp8 = cfg.dtype == "e4m3"
    act = 4 if cfg.dtype == "f32" else 2          # router, combine and residual stay f32/bf16
    el = 1 if fp8 else act                        # expert GEMM operands
    tens = p.get("fp8") if fp8 else p["bf16"]
    tens_sus = p.get("fp8") * p["bf16_sustained"] / p["bf16"] if fp8 else p["bf16_sustained"]
    work = {
        # u and E read, routing (idx + gate) and the load written
        "route": ("hbm", T * d * act + N_r * d * act + R * 8 + N_r * 4,
                  "router: logits GEMM + sigmoid, biased top-K, gates, load, float64 tie-break"),
        # u read once, its K grouped copies written (+ FP8: u quantised first)
        "permute": ("hbm", (T * d * 2 + T * d + T * d // 32 if fp8 else 0) + T * d * el +
                    R * d * el + R * 12 + (R * d // 32 if fp8 else 0),
                    "permute: load scan, stable rank, 16-byte row scatter" +
                    (" (+ 1x128 activation quantiser)" if fp8 else "")),
        "gate_up": ("tensor", 2.0 * Rg * d * 2 * I,
                    ("routed + shared" if merged_shared else "routed") +
                    " gate/up grouped GEMM (tcgen05, fused SwiGLU" +
                    (", E4M3 with per-128 promotion)" if fp8 else ")")),
        "down": ("tensor", 2.0 * Rg * I * d,
                 ("routed + shared" if merged_shared else "routed") +
                 " down grouped GEMM (tcgen05)"),
        "shared": ("tensor", 6.0 * N_s * T * d * I, "shared expert FFNs (tcgen05)"),
        # u, the shared rows and K grouped rows read, h' written
        "combine": ("hbm", T * d * act * (2 + N_s + K) + R * 8,
                    "combine: gate-weighted sum of K grouped rows + shared + residual"),
    }
    out = {}
    for name, (bound, amount, kernel) in work.items():
        ms = phase_ms.get(name)
        if not ms or ms <= 0:
            continue
        if bound == "tensor":
            # the roofline is the slower of the FLOPs at the tensor peak and the
            # algorithmic bytes (weights streamed once, rows in and out) at HBM
            w_groups = {"gate_up": Gw, "down": Gw, "shared": N_s}[name]
            n_rows = {"gate_up": Rg, "down": Rg, "shared": N_s * T}[name]
            per_w = {"gate_up": 2 * I * d, "down": d * I, "shared": 3 * I * d}[name]
            io = {"gate_up": d + I, "down": I + d, "shared": 2 * d}[name]
            nbytes = w_groups * per_w * el + n_rows * io * el
            t_flop = amount / (tens * 1e12)
            t_byte = nbytes / (p["hbm_gbs"] * 1e9)
            ach = amount / (ms / 1e3) / 1e12
            gbs = nbytes / (ms / 1e3) / 1e9
            entry = {"flops_per_launch": amount, "bytes_per_launch": nbytes, "kernel_ms": ms,
                     "tflops": ach, "frac_tensor": ach / tens,
                     "frac_tensor_sustained": ach / tens_sus, "hbm_gbs": gbs,
                     "frac_hbm": gbs / p["hbm_gbs"], "roofline_ms": max(t_flop, t_byte) * 1e3,
                     "tensor_peak_kind": ("measured E4M3 (torch._scaled_mm 8192^3)" if fp8 else
                                          "burst bf16 of " + p["source"]), "kernel": kernel}
            if t_flop >= t_byte:
                entry.update({"bound": "tensor", "achieved": ach, "peak": tens,
                              "unit": "TFLOP/s", "frac": ach / tens})
            else:
                entry.update({"bound": "hbm", "achieved": gbs, "peak": p["hbm_gbs"],
                              "unit": "GB/s", "frac": gbs / p["hbm_gbs"],
                              "peak_kind": "HBM copy bandwidth of " + p["source"]})
            out[name] = entry
        else:
            ach = amount / (ms / 1e3) / 1e9
            out[name] = {"bound": "hbm", "achieved": ach, "peak": p["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / p["hbm_gbs"], "bytes_per_launch": amount, "kernel_ms": ms,
                         "peak_kind": "HBM copy bandwidth of " + p["source"], "kernel": kernel}
    return out


def _load_balance(load_hist, cfg):
    """max/mean expert load of every timed step (mean = T*K/N_r)."""
    h = load_hist.float().cpu()
    r = (h.max(dim=1).values / (cfg.T * cfg.K / cfg.N_r)).tolist()
    return {"max_over_mean_per_step": [round(x, 3) for x in r], "first": round(r[0], 3),
            "last": round(r[-1], 3), "steps": len(r),
            "note": "fresh tokens every step; bias updated after every step (gamma 0.001)"}


def cpu_oracle_sample(cfg, w, n_tokens, seed=0, host=None):
    """Times the C++ CPU oracle on the full route of `n_tokens` sampled tokens
    and their whole layer (expert-major; FP8 configurations quantise each
    touched expert's weights inside the oracle).  Everything the oracle reads
    (the sampled rows, E, b and the weights of every expert the sample
    selects, found by one untimed route) is in host memory before the timer
    starts; `host` (a dict) keeps staged experts across calls.  Returns
    seconds."""
    import numpy as np
    from oracle import moe_ref as R

    host = {} if host is None else host
    rows = np.sort(np.random.default_rng(seed).choice(w["u"].shape[0], n_tokens, replace=False))
    u = w["u"][torch.from_numpy(rows).to(w["u"].device)].cpu()
    if "E" not in host:
        host["E"] = w["E"].cpu()
        host["shared"] = [(w["Ws_gate_up"][j].cpu(), w["Ws_down"][j].cpu())
                          for j in range(cfg.N_s)]
        host["routed"] = {}
    E, shared = host["E"], host["shared"]
    b = w["b"].cpu().numpy()
    G, M = cfg.n_groups, cfg.topk_groups
    touched = np.unique(R.route(u, E, b, cfg.K, G, M)["idx"])
    routed = host["routed"]
    for e in touched:
        if int(e) not in routed:
            routed[int(e)] = (w["W_gate_up"][int(e)].cpu(), w["W_down"][int(e)].cpu())
    t0 = time.perf_counter()
    r = R.route(u, E, b, cfg.K, G, M)
    R.layer_forward(u, r["idx"], r["gate"], routed, shared, fp8=cfg.dtype == "e4m3")
    return time.perf_counter() - t0


def cpu_cores():
    """OpenMP threads the C++ oracle runs with (its default: one per core the
    process may use, unless OMP_NUM_THREADS says otherwise)."""
    from oracle import moe_ref as R
    return R.set_threads(0)


def cpu_model():
    """The host CPU's model name (/proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


# ---------------------------------------------------------------- arms

def run_reference(args, cfg, ws, rank):
    if ws > 1 and rank != 0:
        return
    from mixture_experts_layer_60_b200.synth import make_layer_inputs
    torch.cuda.set_device(0)
    w = make_layer_inputs(cfg, "cuda")
    n_tok = min(args.ref_tokens, cfg.T)
    host = {}
    for _ in range(args.warmup):
        cpu_oracle_sample(cfg, w, n_tok, seed=1, host=host)
    times = [cpu_oracle_sample(cfg, w, n_tok, seed=2 + i, host=host) for i in range(args.steps)]
    tot = sum(times)
    value = n_tok * args.steps / tot
    cores = cpu_cores()
    sample = (f"{n_tok} tokens per step drawn from the {cfg.T}-token batch: full route and "
              f"whole layer (every selected and shared expert) in float64 on the host, C++ "
              f"oracle, weights staged in host memory before the timer")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "N_r": cfg.N_r, "K": cfg.K,
                       "N_s": cfg.N_s, "I": cfg.I, "tokens_per_step": n_tok},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def train_flops(cfg):
    """Algorithmic FLOPs of one training step (forward_train + backward): the
    expert FFNs three times (Fprop, Dgrad, Wgrad), the router logits, and the
    router backward's K-sparse products (d_gate, s, the du term, dE)."""
    ffn = (cfg.K + cfg.N_s) * cfg.T * 6 * cfg.d * cfg.I
    return 3 * ffn + 2 * cfg.T * cfg.d * cfg.N_r + 8 * cfg.T * cfg.K * cfg.d


def measure_train(args, cfg, layer, u, dev, group, p, steps):
    """Times `steps` training steps (forward_train + backward) after 3 warm-up
    steps; the routed expert FFN backward (2 Dgrad + 2 Wgrad grouped GEMMs) is
    timed on its own with events on the same stream."""
    from mixture_experts_layer_60_b200.synth import upstream_grad
    dh = upstream_grad(cfg, dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        layer.forward_train(u)
        layer.backward(dh)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    fb = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if group is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(steps):
        layer.forward_train(u)
        fb[i][0].record(stream)
        layer.backward(dh, ffn_events=ev[i])
        fb[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    bwd_ms = sum(a.elapsed_time(b) for a, b in fb) / steps
    ffn_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    if group is not None:
        tt = torch.tensor([ms, bwd_ms, ffn_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms, bwd_ms, ffn_ms = (float(x) for x in tt)
    ws = dist.get_world_size() if group is not None else 1
    R = cfg.T * cfg.K
    ffn_flops = 12.0 * R * cfg.d * cfg.I
    fp8 = cfg.dtype == "e4m3"
    # the burst figure for a timed region of a few steps; the sustained one beside it
    ratio = (p["fp8"] / p["bf16"]) if fp8 and p.get("fp8") else (2 if fp8 else 1)
    pk = p["bf16"] * ratio
    pk_sus = p["bf16_sustained"] * ratio
    ach = ffn_flops / (ffn_ms / 1e3) / 1e12
    return {
        "metric": "training-step tokens/s (forward keeping activations + backward)",
        "value": cfg.T * ws / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        "backward_ms": bwd_ms, "steps": steps, "warmup": 3,
        "flops_per_step": train_flops(cfg),
        "tflops": train_flops(cfg) / (ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s",
                     "frac": ach / pk, "frac_sustained": ach / pk_sus,
                     "kernel": "routed expert FFN backward (Dgrad down + SwiGLU backward, "
                               "Dgrad gate/up, Wgrad down, Wgrad gate/up; tcgen05" +
                               (", E4M3 operands" if fp8 else "") + ")",
                     "peak_kind": "burst bf16 of " + p["source"] +
                                  ((" x measured E4M3/bf16 ratio" if p.get("fp8") else
                                    " x2 (FP8 nominal ratio)") if fp8 else ""),
                     "kernel_ms": ffn_ms, "flops_per_launch": ffn_flops, "traffic": None},
    }


def run_hbm_kernels(args, cfg, local):
    """The HBM-bound steps alone (route, permute, combine) on T synthetic
    tokens of the configuration's width, with random stand-ins for the
    expert outputs and no expert weights on the device: a right-sized case
    for profiling those kernels.  Prints one JSON line of per-step times."""
    import mixture_experts_layer_60_b200 as moe
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    T, d, N_r, K, N_s = cfg.T, cfg.d, cfg.N_r, cfg.K, cfg.N_s
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    u = torch.randn(T, d, generator=g, device=dev).to(torch.bfloat16)
    E = (torch.randn(N_r, d, generator=g, device=dev) * d ** -0.5).to(torch.bfloat16)
    b = torch.zeros(N_r, device=dev)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    gate = torch.empty(T, K, device=dev)
    counts = torch.empty(N_r, dtype=torch.int32, device=dev)
    rws = torch.empty(moe.moe_route_workspace_size(T, N_r), dtype=torch.uint8, device=dev)
    pws = torch.empty(max(moe.moe_permute_workspace_size(T, N_r), 256), dtype=torch.uint8,
                      device=dev)
    x_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev)
    offsets = torch.empty(N_r + 1, dtype=torch.int32, device=dev)
    perm_src = torch.empty(T * K, dtype=torch.int32, device=dev)
    inv_row = torch.empty(T, K, dtype=torch.int32, device=dev)
    y_perm = torch.randn(T * K, d, generator=g, device=dev).to(torch.bfloat16)
    y_sh = torch.randn(N_s, T, d, generator=g, device=dev).to(torch.bfloat16)
    h = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    names = ("route", "permute", "combine")
    ev = {n: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] for n in names}

    def step(i=None):
        def mark(n, j):
            if i is not None:
                ev[n][i][j].record()
        mark("route", 0)
        moe.moe_route(u, E, b, K, idx, gate, counts, rws)
        mark("route", 1)
        mark("permute", 0)
        moe.moe_permute(u, idx, N_r, x_perm, offsets, perm_src, inv_row, pws)
        mark("permute", 1)
        mark("combine", 0)
        moe.moe_combine(u, y_sh if N_s else None, y_perm, inv_row, gate, h)
        mark("combine", 1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    if moe.moe_device_status() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout")
    ms = {n: sum(a.elapsed_time(c) for a, c in ev[n]) / args.steps for n in names}
    nbytes = {"route": T * d * 2 + N_r * d * 2 + T * K * 8,
              "permute": T * d * 2 * (1 + K) + T * K * 12,
              "combine": T * d * 2 * (2 + N_s + K) + T * K * 8}
    print(json.dumps({"mode": "hbm_kernels", "config": {"workload": cfg.name, "T": T, "d": d,
                                                        "N_r": N_r, "K": K, "N_s": N_s},
                      "ms": ms, "bytes": nbytes,
                      "gbs": {n: nbytes[n] / (ms[n] / 1e3) / 1e9 for n in names}}), flush=True)


def run_ep_emulated(args, cfg, local):
    """Expert parallelism with W ranks emulated on one GPU (each rank keeps
    N_r/W experts and T/W of the tokens): per-phase times of the step and the
    rate of the dispatch and return copy kernels.  On one GPU the rows move
    through this GPU's HBM, not NVLink, so the copy rates are those of the
    kernels, not of the links.  Prints one JSON line."""
    from mixture_experts_layer_60_b200 import moe_device_status
    from mixture_experts_layer_60_b200.parallel_ep import EPGroupEmulated
    from mixture_experts_layer_60_b200.synth import make_layer_inputs, step_u
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    W = args.ep_ranks
    T_r = cfg.T // W
    sub = cfg.with_T(T_r)
    w = make_layer_inputs(sub, dev)
    us = [step_u(sub, s, dev) for s in range(W)]
    grp = EPGroupEmulated(sub, w, W, T_max=T_r, device=dev)
    R = grp.ranks
    stream = torch.cuda.current_stream(dev)

    def phases(ev):
        def mark(name, i):
            if ev is not None:
                ev[name][i].record(stream)
        mark("route_permute", 0)
        for r, u in zip(R, us):
            r.route_permute(u)
        mark("route_permute", 1)
        counts_all = torch.stack([r.counts for r in R])
        mark("plan", 0)
        for r in R:
            r.plan(counts_all)
        mark("plan", 1)
        mark("dispatch", 0)
        for r in R:
            r.dispatch([x.recv_rows for x in R], [x.recv_tags for x in R])
        mark("dispatch", 1)
        mark("experts", 0)
        for r in R:
            r.experts()
        mark("experts", 1)
        mark("return", 0)
        for r in R:
            r.give_back([x.ret_rows for x in R])
        mark("return", 1)
        mark("combine", 0)
        for r in R:
            r.combine()
        mark("combine", 1)

    names = ("route_permute", "plan", "dispatch", "experts", "return", "combine")
    for _ in range(args.warmup):
        phases(None)
    torch.cuda.synchronize()
    evs = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for n in names} for _ in range(args.steps)]
    for i in range(args.steps):
        phases(evs[i])
    torch.cuda.synchronize()
    if moe_device_status() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout")
    ms = {n: sum(e[n][0].elapsed_time(e[n][1]) for e in evs) / args.steps for n in names}
    row_bytes = sub.d * 2
    moved = cfg.T * cfg.K * row_bytes           # every (token, slot) row once
    print(json.dumps({"mode": "ep_emulated", "ranks": W,
                      "config": {"workload": cfg.name, "T": cfg.T, "tokens_per_rank": T_r,
                                 "d": cfg.d, "N_r": cfg.N_r, "experts_per_rank": cfg.N_r // W,
                                 "K": cfg.K, "N_s": cfg.N_s, "I": cfg.I},
                      "ms": ms, "ms_per_step": sum(ms.values()),
                      "tokens_per_s": cfg.T / (sum(ms.values()) / 1e3),
                      "copy_bytes": moved,
                      # row bytes moved per second; the HBM traffic of a copy on one GPU
                      # is twice that (read + write)
                      "dispatch_gbs": moved / (ms["dispatch"] / 1e3) / 1e9,
                      "return_gbs": moved / (ms["return"] / 1e3) / 1e9,
                      "dispatch_hbm_frac": 2 * moved / (ms["dispatch"] / 1e3) / 1e9 /
                                           peaks()["hbm_gbs"],
                      "return_hbm_frac": 2 * moved / (ms["return"] / 1e3) / 1e9 /
                                         peaks()["hbm_gbs"],
                      "note": "ranks emulated on one GPU: dispatch and return copy through "
                              "this GPU's HBM (read + write), not over NVLink"}), flush=True)


def run_ours(args, cfg, ws, rank, local):
    from mixture_experts_layer_60_b200 import moe_device_status
    from mixture_experts_layer_60_b200.layer import MoELayer
    from mixture_experts_layer_60_b200.synth import make_layer_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    p = peaks()
    w = make_layer_inputs(cfg, dev)
    layer = MoELayer(cfg, w, device=dev)
    u = w["u"]
    stream = torch.cuda.current_stream(dev)
    group = dist.group.WORLD if ws > 1 else None
    T_total = cfg.T * ws

    def step(ev=None, u_in=u):
        h = layer.forward(u_in, phase_events=ev)
        if group is not None:
            from mixture_experts_layer_60_b200.parallel_load import allreduce_load
            counts, tt = allreduce_load(layer.counts, cfg.T, group, T_total=T_total)
            layer.bias_update(counts, tt)
        else:
            layer.bias_update()
        return h

    if args.mode == "train":
        if cfg.dtype == "e4m3":
            p["fp8"] = measure_fp8_peak(dev)
        tr = measure_train(args, cfg, layer, u, dev, group, p, args.steps)
        if moe_device_status() != 0:
            raise RuntimeError("a kernel reported a bounded-wait timeout")
        if rank == 0:
            print(json.dumps({**tr, "n_gpus": ws, "dtype": {"bf16": "bf16", "e4m3": "e4m3"}.get(
                cfg.dtype, cfg.dtype), "data": "synthetic",
                              "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d,
                                         "N_r": cfg.N_r, "K": cfg.K, "N_s": cfg.N_s,
                                         "I": cfg.I}}), flush=True)
        return

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if moe_device_status() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout during warm-up")

    # ---- device-resident timed region
    # Multi-step configurations draw fresh tokens every step (generated before
    # the timed region) and record each step's per-expert load.
    multi = cfg.steps > 1
    if multi:
        from mixture_experts_layer_60_b200.synth import step_u
        u_steps = [step_u(cfg, i, dev) for i in range(args.steps)]
        load_hist = torch.empty(args.steps, cfg.N_r, dtype=torch.int32, device=dev)
    ev_pair = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    # phases with a launch of their own (merged shared experts have none)
    phases = [n for n in PHASES if not (n == "shared" and layer.merged_shared)]
    ph_ev = [{name: ev_pair() for name in phases} for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if group is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        if multi:
            step(ph_ev[i], u_in=u_steps[i])
            load_hist[i].copy_(layer.counts)
        else:
            step(ph_ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if group is not None:
        dist.barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    phase_ms = {name: sum(e[name][0].elapsed_time(e[name][1]) for e in ph_ev) / args.steps
                for name in phases}
    if group is not None:
        tt = torch.tensor([ms] + [phase_ms[n] for n in phases], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt[0])
        phase_ms = {n: float(v) for n, v in zip(phases, tt[1:].tolist())}
    gu_ms = phase_ms["gate_up"]
    ms_step = ms / args.steps
    value = cfg.T * ws / (ms_step / 1e3)

    # ---- end to end through the API with host buffers: every step uploads its
    # tokens from pinned host memory and downloads h'; copies run on two copy
    # streams overlapped with the neighbouring steps' compute (HostStepper).
    from mixture_experts_layer_60_b200.hostio import HostStepper
    u_host = u.to("cpu").pin_memory()
    h_hosts = [torch.empty(cfg.T, cfg.d, dtype=u.dtype).pin_memory() for _ in range(2)]
    stepper = HostStepper(cfg.T, cfg.d, u.dtype, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(4, args.steps // 4)

    def host_step(u_in, out):
        layer.forward(u_in, out=out)
        if group is not None:
            from mixture_experts_layer_60_b200.parallel_load import allreduce_load
            counts, tt = allreduce_load(layer.counts, cfg.T, group, T_total=T_total)
            layer.bias_update(counts, tt)
        else:
            layer.bias_update()

    stepper.run([u_host] * 3, [h_hosts[i % 2] for i in range(3)], host_step)   # warm-up
    if group is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    stepper.run([u_host] * e2e_steps, [h_hosts[i % 2] for i in range(e2e_steps)], host_step)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if group is not None:
        tt = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt[0])
    if cfg.dtype == "e4m3":
        p["fp8"] = measure_fp8_peak(dev)
    # ---- training step (bf16 layers): forward keeping activations + backward
    train = None
    if cfg.dtype in ("bf16", "e4m3") and not args.no_train:
        if cfg.d % 256 == 0 and cfg.I % 256 == 0:
            train = measure_train(args, cfg, layer, u, dev, group, p, max(3, args.steps // 4))
        else:
            train = {"skipped": f"the backward needs d and I multiples of 256 (d={cfg.d}, "
                                f"I={cfg.I})"}
    status = moe_device_status()

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if ws == 1 and not args.no_cpu_baseline:
        from oracle import moe_ref as R
        n_tok = min(args.cpu_tokens, cfg.T)
        secs = cpu_oracle_sample(cfg, w, n_tok)
        cpu = {"value": n_tok / secs, "unit": "tokens/s", "cores": cpu_cores(),
               "cpu_model": cpu_model(), "kind": "oracle",
               "sample": f"{n_tok} tokens of the {cfg.T}-token batch, full route + whole layer "
                         f"in float64 by the C++ oracle, weights staged in host memory before "
                         f"the timer ({secs:.1f} s)"}
        if cfg.T <= 4096:
            # the small configurations also on one thread (the same sample)
            n_all = R.set_threads(0)
            R.set_threads(1)
            try:
                secs1 = cpu_oracle_sample(cfg, w, n_tok)
            finally:
                R.set_threads(n_all)
            cpu["one_thread"] = {"value": n_tok / secs1, "unit": "tokens/s", "cores": 1}

    if rank != 0:
        return
    roof_tps, flops, bytes_ = roofline_layer(cfg, p)
    ph = phase_rooflines(cfg, p, phase_ms, layer.merged_shared)
    # dominant kernel: the routed gate/up grouped GEMM.  The timed region is
    # short (well under a second), so the burst peak is the matching
    # denominator; the fraction of the sustained (power-capped) figure is
    # shown beside it.
    roof = dict(ph["gate_up"])
    roof_kernel = roof.pop("kernel")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"f32": "f32", "bf16": "bf16", "e4m3": "e4m3"}[cfg.dtype],
        "data": "synthetic (seeded, random-init weights of the named shape)",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "N_r": cfg.N_r, "K": cfg.K,
                   "N_s": cfg.N_s, "I": cfg.I, "tokens_per_rank": cfg.T,
                   "parallelism": f"dp{ws} (replicas; per-expert load all-reduced)" if ws > 1
                   else "single GPU",
                   "l2": "inputs larger than L2: all expert weights (%.1f GB) stream from HBM "
                         "every step" % (cfg.weight_bytes() / 1e9)},
        "roofline": {**roof, "kernel": roof_kernel, "traffic": measured_traffic(cfg)},
        "phases": ph,
        "layer_roofline": {"tokens_per_s": roof_tps, "frac": value / ws / roof_tps,
                           "flops_per_step": flops, "bytes_per_step": bytes_,
                           "peak_kind": "burst bf16" + (" (FP8: measured E4M3 peak)"
                                                        if cfg.dtype == "e4m3" else "")},
        "clocks": clk,
        "e2e": {"value": cfg.T * ws / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": u.numel() * u.element_size(),
                "d2h_bytes_per_step": u.numel() * u.element_size(),
                "how": "pinned host u uploaded and h' downloaded every step, on two copy "
                       "streams overlapped with the neighbouring steps' compute"},
        "gpu_launches": gpu_launches_per_step(cfg, layer.merged_shared) * args.steps,
        "load_balance": _load_balance(load_hist, cfg) if multi else None,
        "device_status": status,
        "cpu_baseline": cpu,
        "train": train,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="v3_bf16", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=512)
    ap.add_argument("--ref-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-train", action="store_true",
                    help="skip the training-step (forward + backward) measurement")
    ap.add_argument("--mode", default="forward",
                    choices=["forward", "train", "hbm_kernels", "ep_emulated"],
                    help="train: time only training steps and print their line; hbm_kernels: "
                         "route, permute and combine alone (no expert weights), for profiling; "
                         "ep_emulated: expert-parallel phases with --ep-ranks ranks on one GPU")
    ap.add_argument("--ep-ranks", type=int, default=8,
                    help="ep_emulated: ranks emulated on the GPU (each keeps N_r/ranks experts)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="scaled-down variant: tokens per rank (default: the config's T)")
    ap.add_argument("--experts", type=int, default=None,
                    help="scaled-down variant: routed experts (default: the config's N_r)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    cfg = CONFIGS[args.config]
    if args.tokens or args.experts:
        from dataclasses import replace
        T = args.tokens or cfg.T
        N_r = args.experts or cfg.N_r
        cfg = replace(cfg, name=f"{cfg.name}[T={T},N_r={N_r}]", T=T, N_r=N_r)
    ws, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, cfg, ws, rank)
        elif args.mode == "hbm_kernels":
            run_hbm_kernels(args, cfg, local)
        elif args.mode == "ep_emulated":
            run_ep_emulated(args, cfg, local)
        else:
            run_ours(args, cfg, ws, rank, local)
    finally:
        if ws > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
