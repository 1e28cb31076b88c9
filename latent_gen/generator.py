"""Spatio-temporally correlated Q/K/V shaped like video-DiT latents.

Recipe (per (b, h), from its own PCG64 stream seeded with (seed, b, h)):

* 16 frequency triples w_f = (w_t, w_y, w_x) ~ U(0, 0.3);
* a Gaussian map G of shape d x 32;
* per token p = (t, y, x) the 32 features F(p) = [cos(w_f . p), sin(w_f . p)];
* Q = s * G F(p) + 0.3 * N(0,1) and K = s * G F(p) + 0.3 * N(0,1) with
  independent noise, V ~ N(0, 1) (noise and V drawn as float32 normals);
* s is set by bisection so that the standard deviation of q.k / sqrt(d) over
  2^18 seeded token pairs hits the workload's logit std.

Q and K share G, so their logits form a stationary kernel sum_f cos(w_f . dp)
over the spatio-temporal offset dp: nearby tokens in space and time attend to
each other, the latent-space correlation described on the Timeripple and Kaleido
pages (searcharxiv author page, abstracts).  Q and K are formed in fp32, and all three are
rounded to bf16 (round to nearest even).  No step here belongs to the attention method.
"""

from __future__ import annotations

import math
import threading
from concurrent.futures import ThreadPoolExecutor
from typing import Tuple

import numpy as np
import torch

from .configs import Workload

N_PAIRS = 1 << 18


def grid_positions(grid: Tuple[int, int, int]) -> np.ndarray:
    """Integer (t, y, x) coordinates of every token, t-major raster order."""
    T, Y, X = grid
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    return np.stack([t.ravel(), y.ravel(), x.ravel()], axis=1).astype(np.float64)


def _calibrate_scale(U, nq, nk, d, noise, target, rng) -> float:
    n = U.shape[0]
    i = rng.integers(0, n, size=N_PAIRS)
    j = rng.integers(0, n, size=N_PAIRS)
    a = np.empty(N_PAIRS)
    b = np.empty(N_PAIRS)
    c = np.empty(N_PAIRS)
    step = 1 << 14
    for p0 in range(0, N_PAIRS, step):
        ii, jj = i[p0:p0 + step], j[p0:p0 + step]
        ui, uj = U[ii], U[jj]
        qi, kj = nq[ii].astype(np.float64), nk[jj].astype(np.float64)
        a[p0:p0 + step] = np.einsum("pd,pd->p", ui, uj)
        b[p0:p0 + step] = np.einsum("pd,pd->p", ui, kj) + np.einsum("pd,pd->p", qi, uj)
        c[p0:p0 + step] = np.einsum("pd,pd->p", qi, kj)
    inv = 1.0 / math.sqrt(d)

    def std(s: float) -> float:
        return float(np.std((s * s * a + noise * s * b + noise * noise * c) * inv))

    lo, hi = 0.0, 1.0
    while std(hi) < target:
        hi *= 2.0
        if hi > 1e6:
            raise RuntimeError("logit std target unreachable")
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        if std(mid) < target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def make_head(cfg: Workload, b: int, h: int, work=None):
    """fp32 Q, K, V of one (b, h) as numpy arrays [N, d] (before bf16 rounding).

    ``work`` optionally holds reusable float32 buffers (keys "nq", "nk", "v",
    "q", "k") of shape [N, d]; the returned arrays may alias them."""
    N, d = cfg.N, cfg.d
    if work is None:
        work = {}
    for key in ("nq", "nk", "v", "q", "k"):
        if key not in work or work[key].shape != (N, d):
            work[key] = np.empty((N, d), dtype=np.float32)
    rng = np.random.Generator(np.random.PCG64([cfg.seed, b, h]))
    nf = cfg.n_features // 2
    omega = rng.uniform(0.0, 0.3, size=(nf, 3))
    G = rng.standard_normal((cfg.d, cfg.n_features))
    nq, nk, v = work["nq"], work["nk"], work["v"]
    rng.standard_normal(out=nq, dtype=np.float32)
    rng.standard_normal(out=nk, dtype=np.float32)
    rng.standard_normal(out=v, dtype=np.float32)
    phase = grid_positions(cfg.grid) @ omega.T
    F = np.concatenate([np.cos(phase), np.sin(phase)], axis=1)
    U = F @ G.T
    s = _calibrate_scale(U, nq, nk, d, cfg.noise, cfg.logit_std, rng)
    q, k = work["q"], work["k"]
    np.multiply(U, s, out=q, casting="same_kind")
    q += cfg.noise * nq
    np.multiply(U, s, out=k, casting="same_kind")
    k += cfg.noise * nk
    return q, k, v


def make_qkv(cfg: Workload, threads: int = 0):
    """bf16 CPU tensors Q, K, V of shape [B, H, N, d] for workload ``cfg``."""
    B, H, N, d = cfg.B, cfg.H, cfg.N, cfg.d
    Q = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)

    local = threading.local()

    def one(idx):
        b, h = divmod(idx, H)
        if not hasattr(local, "work"):
            local.work = {}
        q, k, v = make_head(cfg, b, h, local.work)
        Q[b, h] = torch.from_numpy(q).to(torch.bfloat16)
        K[b, h] = torch.from_numpy(k).to(torch.bfloat16)
        V[b, h] = torch.from_numpy(v).to(torch.bfloat16)

    n = B * H
    if threads <= 0:
        threads = min(n, 8)
    if threads == 1 or n == 1:
        for idx in range(n):
            one(idx)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(n)))
    return Q, K, V


def make_qkv_steps(cfg: Workload, steps: int, rho: float):
    """A sequence of ``steps`` (Q, K, V) bf16 tensors for successive diffusion
    timesteps that change slowly: step 0 is ``make_qkv(cfg)``; step t mixes the
    previous step with a fresh draw of the same generator (seed shifted by t),
    X_t = bf16(rho X_{t-1} + sqrt(1 - rho^2) Y_t) for each of Q, K, V, which
    keeps every step's distribution and correlates consecutive steps by rho."""
    seq = [make_qkv(cfg)]
    a, b = float(rho), float(np.sqrt(max(0.0, 1.0 - rho * rho)))
    for t in range(1, steps):
        fresh = make_qkv(cfg.with_(seed=cfg.seed + 1000 + t))
        seq.append(tuple((a * x.float() + b * y.float()).to(torch.bfloat16)
                         for x, y in zip(seq[-1], fresh)))
    return seq
