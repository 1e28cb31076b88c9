"""Seeded synthetic inputs shaped like video-DiT attention operands.

This package is shared by the CPU oracle (``oracle/``) and the CUDA path
(``precision_attention_video_b200``).  It holds no arithmetic of the tiered
attention method itself: it only draws Q, K, V and names the workloads.
"""

from .configs import CONFIGS, Workload, get_config  # noqa: F401
from .generator import grid_positions, make_qkv, make_head, make_qkv_steps  # noqa: F401
