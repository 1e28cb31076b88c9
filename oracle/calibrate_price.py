"""Calibrate the single price of the price-router workload on the oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``): run once to write
``latent_gen/price.json``; nothing imports this module.

The workload is the 480p-video-like layer (B=1, H=40, N=32760, d=128,
128 x 128 tiles) with all four tiers (bf16, NVFP4 + residual, NVFP4, skip)
chosen by the price rule of ``oracle.route`` ("Triage" abstract: a single
price sets the trade-off between predicted error and compute), with the
rule's default tier costs (each tier's per-tile time on the fused kernel
relative to a bf16 tile).  Reading: one
global price, found by bisection on the oracle's fp64 pooled masses and skip
spreads of all heads, so that half of all tiles are skipped (the forced
diagonal counts as kept), the share the pooled-mass 480p workload skips.

    python -m oracle.calibrate_price
"""

from __future__ import annotations

import json
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from latent_gen import get_config  # noqa: E402
from latent_gen.generator import make_head  # noqa: E402
from oracle.quant import LOW_NVFP4_RES  # noqa: E402
from oracle.route import (TIER_FULL, TIER_LOW, TIER_RES, TIER_SKIP,  # noqa: E402
                          assign_tiers_price, block_spread, default_tier_cost, diag_blocks,
                          pool_means, pooled_mass)

TARGET_SKIP = 0.5


def head_stats(cfg):
    out = []
    scale = 1.0 / math.sqrt(cfg.d)
    for h in range(cfg.H):
        q, k, _ = make_head(cfg, 0, h)
        Qh = torch.from_numpy(q).to(torch.bfloat16).double().numpy()
        Kh = torch.from_numpy(k).to(torch.bfloat16).double().numpy()
        qbar, _ = pool_means(Qh, cfg.block_q)
        kbar, n_k = pool_means(Kh, cfg.block_k)
        M = pooled_mass(qbar, kbar, n_k, scale)
        qvar = block_spread(Qh, cfg.block_q)
        delta = scale * np.sqrt((qbar * qbar + qvar) @ block_spread(Kh, cfg.block_k).T)
        out.append((M, delta))
        print("head", h, flush=True)
    return out


def fractions(stats, cfg, price):
    counts = np.zeros(4)
    for M, delta in stats:
        for i in range(M.shape[0]):
            t, _ = assign_tiers_price(M[i], delta[i], price, LOW_NVFP4_RES,
                                      diag_blocks(i, cfg.block_q, cfg.block_k, cfg.N))
            counts += np.bincount(t, minlength=4)
    return counts / counts.sum()


def main():
    cfg = get_config("480p-price")
    stats = head_stats(cfg)
    lo, hi = 0.0, 1.0          # the skipped share grows with the price
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if fractions(stats, cfg, mid)[TIER_SKIP] < TARGET_SKIP:
            lo = mid
        else:
            hi = mid
    price = 0.5 * (lo + hi)
    f = fractions(stats, cfg, price)
    out = {"workload": "480p-video-like, price router, NVFP4 + residual", "target_skip": TARGET_SKIP,
           "method": "bisection on the oracle's fp64 pooled masses and skip spreads (all 40 heads)",
           "tier_cost": list(default_tier_cost(LOW_NVFP4_RES)),
           "price": price,
           "achieved": {"full": f[TIER_FULL], "res": f[TIER_RES], "low": f[TIER_LOW], "skip": f[TIER_SKIP]}}
    print(out, flush=True)
    path = os.path.join(ROOT, "latent_gen", "price.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
