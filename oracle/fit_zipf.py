"""Fits the centroid norms of the skewed-load input recipe (test/input tooling).

    python -m oracle.fit_zipf  [writes mixture_experts_layer_60_b200/data/zipf_lambda_v3.json]

The skewed V3 configuration rescales each expert centroid to a norm lambda_i
(e_i <- lambda_i e_i / |e_i|).  For tokens u ~ N(0, I) the logit u.e_i is then
lambda_i z_i with z_i ~ N(0, 1), nearly independent across experts (random
centroids in 7168 dimensions are almost orthogonal).  Expert i should be
selected (top-K of Sigmoid(logit) + b with b = 0) with probability
pi_i = min(1, c (i+1)^-1.2), c such that sum_i pi_i = K: a Zipf(1.2)
popularity, clipped because no expert can be in more than every token's
selection.  Norms alone cannot push an expert above ~1/2 popularity (its logit
is negative for half the tokens), so the fit is a best effort: the achieved
popularity is recorded next to lambda and reported, not asserted.

The fit is a damped fixed-point iteration lambda_i <- lambda_i (pi_i / p_i)^0.25,
rescaled so the largest norm stays at LAM_MAX, on a seeded calibration batch, where p_i is the selection rate the oracle's own
sigmoid and biased top-K produce; it runs once and its output is data.
"""
from __future__ import annotations

import json
import os

import numpy as np

from . import moe_oracle as O

N_R, K, ZIPF, SEED = 256, 8, 1.2, 2
CALIB_TOKENS, ITERS, STEP = 8192, 150, 0.25
# Norms above ~5 would push float32 sigmoids to exactly 1.0 for many tokens, and
# ties among saturated scores would then be settled by expert index, not by norm.
LAM_MIN, LAM_MAX = 0.02, 5.0
OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mixture_experts_layer_60_b200", "data", "zipf_lambda_v3.json")


def zipf_target(n=N_R, k=K, a=ZIPF):
    w = np.arange(1, n + 1, dtype=np.float64) ** -a
    lo, hi = 0.0, 1e6
    for _ in range(200):                      # bisection on c: sum min(1, c w) = k
        c = 0.5 * (lo + hi)
        if np.minimum(1.0, c * w).sum() > k:
            hi = c
        else:
            lo = c
    return np.minimum(1.0, lo * w)


def selection_rate(lam, z):
    # logits lam_i z_{t,i}: the affinity of u = z against centroids diag(lam)
    s = O.affinity(z, np.diag(lam))
    idx, _ = O.biased_topk(s, np.zeros(len(lam), np.float32), K)
    return O.load_counts(idx, len(lam)) / z.shape[0]


def fit():
    rng = np.random.default_rng(SEED)
    z = rng.standard_normal((CALIB_TOKENS, N_R))
    pi = zipf_target()
    lam = np.ones(N_R)
    for _ in range(ITERS):
        p = np.maximum(selection_rate(lam, z), 0.5 / CALIB_TOKENS)
        lam = lam * (pi / p) ** STEP
        # only ratios of norms matter: pin the largest at LAM_MAX
        lam = np.clip(lam * (LAM_MAX / lam.max()), LAM_MIN, LAM_MAX)
    p = selection_rate(lam, rng.standard_normal((CALIB_TOKENS, N_R)))
    return lam, pi, p


def main():
    lam, pi, p = fit()
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    with open(OUT, "w") as f:
        json.dump({"recipe": "centroid norms for Zipf(1.2) expert popularity, N_r=256, K=8; "
                             "written by oracle/fit_zipf.py",
                   "lambda": [round(float(x), 6) for x in lam],
                   "target_popularity": [round(float(x), 6) for x in pi],
                   "achieved_popularity_calibration": [round(float(x), 6) for x in p],
                   "achieved_max_over_mean_load": round(float(p.max() / (K / N_R)), 3)},
                  f, indent=1)
    print(f"wrote {OUT}: max/mean load {p.max() / (K / N_R):.2f}, "
          f"top-5 popularity {np.round(p[:5], 3).tolist()}")


if __name__ == "__main__":
    main()
