"""Seeded synthetic inputs for the layer (no layer arithmetic lives here).

Recipe, per configuration (one torch.Generator on the target device, seeded
with the configuration's seed, drawn in this fixed order):

  1. u      [T, d]          N(0, 1)                          (C5: then x50 on a Bernoulli(0.001) mask, drawn last)
  2. E      [N_r, d]        N(0, 1/d)   expert centroids e_i
  3. b      [N_r]           0, or U(-0.01, 0.01)
  4. W_gate [N_r][I, d]     N(0, 1/d)   expert by expert
  5. W_up   [N_r][I, d]     N(0, 1/d)
  6. W_down [N_r][d, I]     N(0, 1/I)
  7. shared experts: W_gate, W_up, W_down the same way, N_s of each
  8. outlier mask (only when outlier_frac > 0)

Every value is drawn in float32 and rounded once to the storage dtype (float32
for the tiny configuration, bfloat16 otherwise; the FP8 configuration stores
bfloat16 and is quantised by the library).  Routed and shared gate/up weights
are stored stacked as W_gate_up [G, 2I, d]: rows [0, I) hold W_gate and rows
[I, 2I) hold W_up.

Skewed-load configurations rescale the centroids to e_i <- lambda_i e_i / |e_i|
with a fitted lambda (popularity data, supplied by the caller), and draw a fresh
u for every step s from the seed 1_000_000 * seed + s + 1.
"""
from __future__ import annotations

import torch

from .configs import LayerConfig


def storage_dtype(cfg: LayerConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def _normal(gen, shape, std, device, dtype):
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def zipf_lambda_v3():
    """Centroid norms of the skewed-load V3 recipe (fitted once, stored as data;
    see data/zipf_lambda_v3.json for the target and achieved popularity)."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "data", "zipf_lambda_v3.json")
    with open(path) as f:
        return json.load(f)["lambda"]


def make_layer_inputs(cfg: LayerConfig, device="cuda", T: int | None = None,
                      zipf_lambda=None) -> dict:
    """All tensors of one configuration, generated on `device`.

    T overrides the token count (the weights are unchanged: they are drawn
    after u, and u's draw count depends on T, so a different T yields a
    different, equally valid, sample of the same recipe)."""
    T = cfg.T if T is None else T
    dt = storage_dtype(cfg)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    d, N_r, I, N_s = cfg.d, cfg.N_r, cfg.I, cfg.N_s
    out = {}
    u32 = torch.randn(T, d, generator=gen, device=device, dtype=torch.float32)
    out["E"] = _normal(gen, (N_r, d), d ** -0.5, device, torch.float32)
    if cfg.bias == "uniform":
        b = (torch.rand(N_r, generator=gen, device=device, dtype=torch.float32) * 2 - 1) * 0.01
    else:
        b = torch.zeros(N_r, device=device, dtype=torch.float32)
    out["b"] = b

    def experts(G):
        wgu = torch.empty(G, 2 * I, d, device=device, dtype=dt)
        wdn = torch.empty(G, d, I, device=device, dtype=dt)
        for e in range(G):
            wgu[e, :I] = _normal(gen, (I, d), d ** -0.5, device, dt)
        for e in range(G):
            wgu[e, I:] = _normal(gen, (I, d), d ** -0.5, device, dt)
        for e in range(G):
            wdn[e] = _normal(gen, (d, I), I ** -0.5, device, dt)
        return wgu, wdn

    out["W_gate_up"], out["W_down"] = experts(N_r)
    out["Ws_gate_up"], out["Ws_down"] = experts(N_s)
    if cfg.outlier_frac > 0:
        mask = torch.rand(T, d, generator=gen, device=device) < cfg.outlier_frac
        u32 = torch.where(mask, u32 * cfg.outlier_scale, u32)
    out["u"] = u32.to(dt)
    if zipf_lambda is None and cfg.zipf > 0:
        zipf_lambda = zipf_lambda_v3()
    if zipf_lambda is not None:
        lam = torch.as_tensor(zipf_lambda, dtype=torch.float32, device=device)
        E = out["E"]
        out["E"] = E / E.norm(dim=1, keepdim=True) * lam[:, None]
    out["E"] = out["E"].to(dt)
    return out


def step_u(cfg: LayerConfig, step: int, device="cuda", T: int | None = None) -> torch.Tensor:
    """Fresh tokens for step `step` of a multi-step run."""
    T = cfg.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed(1_000_000 * cfg.seed + step + 1)
    return torch.randn(T, cfg.d, generator=gen, device=device,
                       dtype=torch.float32).to(storage_dtype(cfg))


def upstream_grad(cfg: LayerConfig, device="cuda", T: int | None = None,
                  step: int = 0) -> torch.Tensor:
    """Upstream gradient dL/dh' [T, d] for a backward: N(0, 1/d) from the seed
    2_000_000 * seed + step + 1, rounded once to the storage dtype."""
    T = cfg.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed(2_000_000 * cfg.seed + step + 1)
    return _normal(gen, (T, cfg.d), cfg.d ** -0.5, device, storage_dtype(cfg))
