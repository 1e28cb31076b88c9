"""Tiered-precision block-sparse attention for video diffusion transformers on B200.

The compute path is libtiered_attn.so (hand-written sm_100a CUDA kernels
behind a C ABI, see include/tiered_attn.h); this package is its thin Python
binding.  The library is built in-tree by ``python -m
precision_attention_video_b200.build`` and loaded on the first call; a call
without it raises ImportError (there is no fallback path).
"""

from .binding import (  # noqa: F401
    TA_OK, TA_ERR_INVALID_ARG, TA_ERR_UNSUPPORTED, TA_ERR_WORKSPACE, TA_ERR_CUDA, TA_ERR_TIMEOUT,
    TA_LOW_NONE, TA_LOW_FP8_E4M3, TA_LOW_NVFP4, TA_LOW_NVFP4_RES,
    TA_TIER_SKIP, TA_TIER_LOW, TA_TIER_RES, TA_TIER_FULL, TA_DEBUG_DROP_FIRST_K,
    TieredAttnError, alloc_workspace, forward, get_status, layer_from_host, make_params,
    params_for, plan, plan_views, prep, route, route_noalloc, status_string, version,
    workspace_bytes,
)
from .binding import LIB_PATH  # noqa: F401
