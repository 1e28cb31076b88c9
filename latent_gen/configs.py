"""Workload definitions for tiered-precision video-DiT attention.

Each workload fixes the attention shape (B, H, N, d), the latent grid the N
tokens are rastered from (t-major: token = (t*Y + y)*X + x), the tile shape,
the low-precision format and the cumulative-mass thresholds.

Shapes follow the video-DiT settings discussed in "Triage" (zhuanzhiai paper
page, abstract: tens of thousands of visual tokens, NVFP4 skim / refine tiers)
and "FG-Attn" (searcharxiv author page, abstract: 70% sparsity point).  The
sweep thresholds are calibrated on the oracle's pooled masses by
``oracle/calibrate_sweep.py`` and stored in ``sweep_tau.json`` beside this file.
"""

from __future__ import annotations

import json
import os
from dataclasses import dataclass, field, replace
from typing import Dict, Tuple

# Low-precision formats (same numbering as the C ABI's ta_low_format).
LOW_NONE = 0
LOW_FP8 = 1
LOW_NVFP4 = 2
LOW_NVFP4_RES = 3

LOW_NAMES = {LOW_NONE: "none", LOW_FP8: "fp8_e4m3", LOW_NVFP4: "nvfp4",
             LOW_NVFP4_RES: "nvfp4+residual"}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: Tuple[int, int, int]          # (T, Y, X) latent grid, t-major raster
    block_q: int
    block_k: int
    logit_std: float                    # target std of q.k/sqrt(d) over token pairs
    low: int                            # LOW_* format of the low tier
    tau: Tuple[float, ...]              # ascending thresholds: full, [res], low
    p_offset_log2: int                  # power-of-two offset carried by P' = 2^o e^(s-m)
    seed: int = 0
    noise: float = 0.3                  # std of the i.i.d. noise added to Q and K
    n_features: int = 32                # cos/sin Fourier features per token
    keep_diag_full: int = 1
    router: int = 0                     # 0: pooled-mass thresholds tau; 1: single price; 2: entropy
    price: float = 0.0                  # the price of router 1
    kappa: float = 1.0                  # the retention scale of router 2
    tier_cost: Tuple[float, ...] = (0.0, 0.0, 0.0, 0.0)   # router 1's costs by tier code; 0s: defaults
    extra: Dict[str, float] = field(default_factory=dict)

    @property
    def N(self) -> int:
        t, y, x = self.grid
        return t * y * x

    @property
    def n_qb(self) -> int:
        return -(-self.N // self.block_q)

    @property
    def n_kb(self) -> int:
        return -(-self.N // self.block_k)

    @property
    def key_pack(self) -> int:
        """Key blocks per attention tile: 32-key blocks go four to a 128-key tile."""
        return 4 if self.block_k == 32 else 1

    def dense_flops(self) -> float:
        """Dense-equivalent attention FLOPs: 4*B*H*N^2*d (QK^T and PV)."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _sweep_tau() -> Dict[str, Tuple[float, float]]:
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sweep_tau.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        raw = json.load(f)
    return {k: tuple(v["tau"]) for k, v in raw["points"].items()}


def _price() -> float:
    """The price-router workload's price (written by oracle/calibrate_price.py)."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "price.json")
    if not os.path.exists(path):
        return 0.0
    with open(path) as f:
        return float(json.load(f)["price"])


def _kappa() -> float:
    """The entropy-router workload's retention scale (written by
    oracle/calibrate_entropy.py)."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kappa.json")
    if not os.path.exists(path):
        return 1.0
    with open(path) as f:
        return float(json.load(f)["kappa"])


def _build() -> Dict[str, Workload]:
    c: Dict[str, Workload] = {}
    c["tiny"] = Workload("tiny", 1, 2, 64, (4, 16, 16), 64, 64, 3.0, LOW_FP8,
                         (0.7, 0.95), p_offset_log2=8)
    c["small"] = Workload("small", 1, 12, 64, (8, 32, 32), 128, 64, 3.0, LOW_FP8,
                          (0.6, 0.9), p_offset_log2=8)
    c["480p"] = Workload("480p", 1, 40, 128, (21, 30, 52), 128, 128, 4.0, LOW_NVFP4,
                         (0.6, 0.9), p_offset_log2=11)
    # Four tiers: full below 0.5, NVFP4+residual on the middle-mass half up to
    # 0.675, NVFP4 up to 0.85, skip beyond.
    c["720p"] = Workload("720p", 1, 24, 128, (33, 45, 80), 128, 128, 4.0, LOW_NVFP4_RES,
                         (0.5, 0.675, 0.85), p_offset_log2=11)
    # The 480p shape with all four tiers chosen by the single-price router;
    # the price is calibrated on the oracle for half of the tiles skipped.
    c["480p-price"] = Workload("480p-price", 1, 40, 128, (21, 30, 52), 128, 128, 4.0,
                               LOW_NVFP4_RES, (0.5, 0.675, 0.85), p_offset_log2=11,
                               router=1, price=_price())
    # The 480p layer with the kept blocks of each query block chosen from the
    # entropy of its pooled pattern; kappa calibrated on the oracle for half
    # of the tiles skipped.
    c["480p-entropy"] = Workload("480p-entropy", 1, 40, 128, (21, 30, 52), 128, 128, 4.0,
                                 LOW_NVFP4, (0.6, 0.9), p_offset_log2=11, router=2,
                                 kappa=_kappa())
    # The 480p layer routed at 32-key granularity ("FG-Attn", searcharxiv
    # author page, abstract: skipping at M x N sub-tiles, M >= 16, N >= 1;
    # here M = 128 queries, N = 32 keys); the attention kernel packs four kept
    # 32-key blocks of one tier into each 128-key tile.
    c["480p-fg"] = Workload("480p-fg", 1, 40, 128, (21, 30, 52), 128, 32, 4.0, LOW_NVFP4,
                            (0.6, 0.9), p_offset_log2=11)
    # Sparsity sweep on the 480p shape with an FP8 low tier; the 0% point runs
    # every tile in bf16 (thresholds above every cumulative mass).
    sweep = _sweep_tau()
    for pct in (0, 30, 50, 70, 90):
        name = f"sweep{pct}"
        if pct == 0:
            tau = (2.0, 2.0)
        else:
            tau = sweep.get(name, (0.0, 0.0))
        c[name] = Workload(name, 1, 40, 128, (21, 30, 52), 128, 128, 4.0, LOW_FP8,
                           tau, p_offset_log2=8, extra={"skip_pct": float(pct)})
    return c


CONFIGS: Dict[str, Workload] = _build()


def get_config(name: str) -> Workload:
    try:
        return CONFIGS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}") from None
