"""Naive fp64 softmax attention (oracle pin, not the method).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

O = softmax(Q K^T * scale) V row by row, with the row max subtracted before
the exponential.  It is the dense self-attention that the video-DiT pages
("Triage", "FG-Attn", "HierPAS" abstracts) approximate.
"""

from __future__ import annotations

import math

import numpy as np


def dense_attention(Qh: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, scale: float = 0.0):
    d = Qh.shape[-1]
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    s = (Qh @ Kh.T) * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ Vh) / p.sum(axis=1, keepdims=True)
