"""CPU oracle for tiered-precision block-sparse video-DiT attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) may import or call this package; only the tests, the smoke
check and the benchmark's CPU-baseline leg do.  It shares no code with the GPU
path; both read the same seeded inputs from ``latent_gen``.

It is a plain, slow, step-by-step restatement of the method in fp64, with the
low-precision formats rounded in software:

* ``formats``   bf16 / fp32 / FP8 e4m3 / FP4 e2m1 / ue4m3 rounding and codes;
* ``quant``     per-tile FP8 and per-16 NVFP4 (+ residual) copies of Q, K, V;
* ``route``     block pooling, pooled block softmax, cumulative-mass tiers or
                the price rule, their flags and per-row tile lists;
* ``attention`` the one-pass online-softmax attention over the tiers;
* ``dense``     naive fp64 softmax attention (a pin, not the method).

The method is the one on the "Triage" page (zhuanzhiai paper page, abstract):
each (query-block, key-block) tile is skipped and replaced by its block means,
skimmed in NVFP4, or refined with an NVFP4 residual correction, with a router
working from block statistics; tiers of progressively reduced precision follow
"HierPAS" (conference listing, abstract) and two thresholds on attention
probability follow "APT" (Lattice paper summary, APDT).  Every step the pages
leave open is a stated reading; each function's docstring names it.
"""

from .formats import (  # noqa: F401
    bf16_rne, fp32_rne, e4m3_round, e4m3_encode, e4m3_decode,
    e2m1_round, e2m1_encode, e2m1_decode, ue4m3_encode, ue4m3_decode,
)
from .quant import (  # noqa: F401
    fp8_tile_scale, quant_fp8_tiles, nvfp4_quant_groups, quant_nvfp4_rows,
    quant_nvfp4_cols, dequant_nvfp4_rows, dequant_nvfp4_cols, quantize_head,
)
from .route import (  # noqa: F401
    pool_means, pooled_mass, diag_blocks, assign_tiers, row_lists, route_head,
    block_spread, price_tiers, assign_tiers_price, reuse_plan, assign_tiers_entropy,
    ROUTER_MASS, ROUTER_PRICE, ROUTER_ENTROPY,
    TIER_SKIP, TIER_LOW, TIER_RES, TIER_FULL,
)
from .attention import tiered_attention_head, tiered_attention  # noqa: F401
from .dense import dense_attention  # noqa: F401
