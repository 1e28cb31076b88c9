"""Calibrate the retention scale of the entropy-router workload on the oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``): run once to write
``latent_gen/kappa.json``; nothing imports this module.

The workload is the 480p-video-like layer (B=1, H=40, N=32760, d=128,
128 x 128 tiles, NVFP4 low tier, tau 0.6 / 0.9 for precision) with the kept
blocks of each query block chosen by the entropy rule of ``oracle.route``
("HierPAS" abstract: retention ratios from an entropy analysis of a cheap
attention-pattern estimate).  Reading: one global retention scale kappa,
found by bisection on the oracle's fp64 pooled masses of all heads, so that
half of all tiles are skipped (the forced diagonal counts as kept), the share
the pooled-mass 480p workload skips.

    python -m oracle.calibrate_entropy
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
from oracle.route import (TIER_FULL, TIER_LOW, TIER_RES, TIER_SKIP,  # noqa: E402
                          assign_tiers_entropy, diag_blocks, pool_means, pooled_mass)

TARGET_SKIP = 0.5


def head_masses(cfg):
    out = []
    for h in range(cfg.H):
        q, k, _ = make_head(cfg, 0, h)
        Qh = torch.from_numpy(q).to(torch.bfloat16).double().numpy()
        Kh = torch.from_numpy(k).to(torch.bfloat16).double().numpy()
        qbar, _ = pool_means(Qh, cfg.block_q)
        kbar, n_k = pool_means(Kh, cfg.block_k)
        out.append(pooled_mass(qbar, kbar, n_k, 1.0 / math.sqrt(cfg.d)))
    return out


def fractions(masses, cfg, kappa):
    counts = np.zeros(4)
    for M in masses:
        for i in range(M.shape[0]):
            t, _, _ = assign_tiers_entropy(M[i], cfg.tau, kappa,
                                           diag_blocks(i, cfg.block_q, cfg.block_k, cfg.N))
            counts += np.bincount(t, minlength=4)
    return counts / counts.sum()


def main():
    cfg = get_config("480p-entropy")
    masses = head_masses(cfg)
    lo, hi = 0.0, 4.0          # the skipped share falls as kappa grows
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if fractions(masses, cfg, mid)[TIER_SKIP] > TARGET_SKIP:
            lo = mid
        else:
            hi = mid
    kappa = 0.5 * (lo + hi)
    f = fractions(masses, cfg, kappa)
    out = {"workload": "480p-video-like, entropy router, NVFP4", "target_skip": TARGET_SKIP,
           "method": "bisection on the oracle's fp64 pooled masses (all 40 heads)",
           "kappa": kappa,
           "achieved": {"full": f[TIER_FULL], "res": f[TIER_RES], "low": f[TIER_LOW], "skip": f[TIER_SKIP]}}
    print(out, flush=True)
    path = os.path.join(ROOT, "latent_gen", "kappa.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
