"""Calibrate the sparsity-sweep thresholds on the oracle's pooled masses.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``): run once to write
``latent_gen/sweep_tau.json``; nothing imports this module.

The sweep runs the 480p-video-like layer (B=1, H=40, N=32760, d=128,
128 x 128 tiles, FP8 low tier) at skip fractions 30/50/70/90 % with FP8 low
tiles fixed at 20 % of the kept tiles; the 0 % point keeps every tile full.
"FG-Attn" (searcharxiv author page, abstract) quotes its kernel speedup at 70 %
sparsity.  Reading: one global (tau_full, tau_low) pair per point, found by
bisection on the oracle's fp64 pooled masses of all heads: first tau_low so
that the skipped share of all tiles (the forced diagonal counts as kept) hits
the target, then tau_full in [0, tau_low] so that low tiles are 20 % of the
kept ones.  The achieved fractions are stored beside the thresholds.

    python -m oracle.calibrate_sweep
"""

from __future__ import annotations

import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from latent_gen import get_config  # noqa: E402
from latent_gen.generator import make_head  # noqa: E402
from oracle.route import (TIER_FULL, TIER_LOW, TIER_SKIP, assign_tiers, diag_blocks,  # noqa: E402
                          pool_means, pooled_mass)

TARGETS = (30, 50, 70, 90)
LOW_SHARE = 0.2


def head_masses(cfg):
    out = []
    for h in range(cfg.H):
        q, k, _ = make_head(cfg, 0, h)
        Qh = torch.from_numpy(q).to(torch.bfloat16).double().numpy()
        Kh = torch.from_numpy(k).to(torch.bfloat16).double().numpy()
        qbar, _ = pool_means(Qh, cfg.block_q)
        kbar, n_k = pool_means(Kh, cfg.block_k)
        out.append(pooled_mass(qbar, kbar, n_k, 1.0 / np.sqrt(cfg.d)))
    return out


def fractions(masses, cfg, tau):
    counts = np.zeros(4)
    for M in masses:
        for i in range(M.shape[0]):
            t, _ = assign_tiers(M[i], tau, diag_blocks(i, cfg.block_q, cfg.block_k, cfg.N))
            counts[TIER_FULL] += np.sum(t == TIER_FULL)
            counts[TIER_LOW] += np.sum(t == TIER_LOW)
            counts[TIER_SKIP] += np.sum(t == TIER_SKIP)
    total = counts.sum()
    return counts[TIER_FULL] / total, counts[TIER_LOW] / total, counts[TIER_SKIP] / total


def bisect(f, lo, hi, target, increasing, iters=30):
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        v = f(mid)
        if (v < target) == increasing:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def main():
    cfg = get_config("sweep70")
    masses = head_masses(cfg)
    points = {}
    for pct in TARGETS:
        target = pct / 100.0
        # skip fraction falls as tau_low grows (every tile below it is kept)
        tau_low = bisect(lambda x: -fractions(masses, cfg, (0.0, x))[2], 0.0, 1.0, -target, True)
        def low_share(x):
            full, low, _ = fractions(masses, cfg, (x, tau_low))
            return low / (full + low)
        tau_full = bisect(low_share, 0.0, tau_low, LOW_SHARE, False)
        full, low, skip = fractions(masses, cfg, (tau_full, tau_low))
        points[f"sweep{pct}"] = {"tau": [tau_full, tau_low],
                                 "achieved": {"full": full, "low": low, "skip": skip,
                                              "low_share_of_kept": low / (full + low)}}
        print(pct, points[f"sweep{pct}"], flush=True)
    out = {"workload": "480p-video-like, FP8 low tier", "low_share_target": LOW_SHARE,
           "method": "bisection on the oracle's fp64 pooled masses (all 40 heads)",
           "points": points}
    path = os.path.join(ROOT, "latent_gen", "sweep_tau.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
