"""One-pass online-softmax attention over tiered tiles (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pass follows "Triage" (zhuanzhiai paper page, abstract): all three tiers
run in a single pass; a skipped tile is replaced by its block means, so block
j of n_j keys adds n_j exp(q . kbar_j * scale) to the softmax denominator and
that weight times vbar_j to the numerator.  Kept tiles are computed in bf16
(full), FP8 / NVFP4 (low) or NVFP4 plus an NVFP4 residual (refine).

Per query block i (all its rows together; every row of a block shares the
block's tile list), in fp64, starting from m = -inf, l = 0, acc = 0:

* kept tiles in list order (full, then residual, then low; within a tier by
  descending pooled mass, lower j first on ties):
    s      = logits of the tile's real keys from the tier's operands * scale
             full: bf16 Q . bf16 K;  low: deq(Q^) . deq(K^);
             residual: deq(Q1)deq(K1) + deq(Q1)deq(K2) + deq(Q2)deq(K1)
    m'     = max(m, max s);  l, acc *= exp(m - m')
    P'     = 2^o exp(s - m')           (o = p_offset_log2: a power of two
                                        carried by numerator and denominator
                                        alike, so it cancels in O; it lifts P'
                                        into the FP8 / FP4 grids)
    l     += sum P'                    (unquantised P')
    acc   += q(P') V_tier              full: bf16(P') V;  FP8: e4m3(P') deq(V^);
                                       NVFP4: nvfp4_16keys(P') deq(V^);
                                       residual: P1 V1 + P1 V2 + P2 V1 with
                                       P1 = nvfp4(P'), P2 = nvfp4(fp32(P' - P1))
* skipped blocks, as one group (order immaterial):
    s_j = q . bf16(kbar_j) * scale;  m' = max(m, max_j s_j); rescale
    w_j = n_j 2^o exp(s_j - m');  l += sum w_j;  acc += bf16(w_j) bf16(vbar_j)
* O = acc / l.

Finer key granularity ("FG-Attn", searcharxiv author page, abstract: skip
score computation at M x N sub-tiles, M >= 16 queries, N >= 1 keys): with
narrow key blocks (block_k = 32) the kept blocks of one tier are taken
``key_pack`` at a time in list order, their keys side by side, as one tile:
one running-max update per tile, NVFP4 groups of P' starting at each block's
first key (a block's real keys only), skipped blocks unchanged.

Readings: the tier order (full, residual, low, skip) and the descending-mass
order inside a tier put the running max near its final value before any P'
is quantised; the denominator sums P' before
quantisation; the skipped blocks of a row enter as one group with a single
running-max update.  ``exact=True`` turns off every rounding of P' and w (the
operand copies stay quantised); the pins use it.
"""

from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .formats import bf16_rne, e4m3_round, fp32_rne
from .quant import (LOW_FP8, LOW_NONE, LOW_NVFP4, LOW_NVFP4_RES, nvfp4_dequant_groups,
                    nvfp4_quant_groups, quantize_head)
from .route import TIER_FULL, TIER_LOW, TIER_RES, route_head


def nvfp4_along_keys(P: np.ndarray) -> np.ndarray:
    """NVFP4 round trip of P [rows, nk] with groups of 16 keys from the tile start."""
    rows, nk = P.shape
    npad = -(-nk // 16) * 16
    Pp = np.zeros((rows, npad))
    Pp[:, :nk] = P
    codes, sc = nvfp4_quant_groups(Pp.reshape(rows, npad // 16, 16))
    return nvfp4_dequant_groups(codes, sc).reshape(rows, npad)[:, :nk]


def _qblock(i, Qh, Kh, Vh, rt, qt, low, Bq, Bk, o, scale, exact, pack):
    N = Qh.shape[0]
    r0, r1 = i * Bq, min(N, (i + 1) * Bq)
    q = Qh[r0:r1]
    nr, d = q.shape
    m = np.full(nr, -np.inf)
    l = np.zeros(nr)
    acc = np.zeros((nr, d))
    two_o = 2.0 ** o
    counts = rt["counts"][i]
    lst = rt["lists"][i]
    pos = 0
    for tier, cnt in ((TIER_FULL, counts[0]), (TIER_RES, counts[1]), (TIER_LOW, counts[2])):
        tier_blocks = lst[pos:pos + cnt]
        for g0 in range(0, cnt, pack):
            # one tile: `pack` consecutive list entries of the tier, their
            # keys side by side (segments in list order)
            segs = [(j * Bk, min(N, (j + 1) * Bk)) for j in tier_blocks[g0:g0 + pack]]
            keys = np.concatenate([np.arange(k0, k1) for k0, k1 in segs])
            cuts = np.cumsum([0] + [k1 - k0 for k0, k1 in segs])
            if tier == TIER_FULL:
                s = (q @ Kh[keys].T) * scale
            elif tier == TIER_LOW:
                s = (qt["dq"][r0:r1] @ qt["dk"][keys].T) * scale
            else:
                a1, a2 = qt["dq"][r0:r1], qt["rq"][r0:r1]
                b1, b2 = qt["dk"][keys], qt["rk"][keys]
                s = (a1 @ b1.T + a1 @ b2.T + a2 @ b1.T) * scale
            m_new = np.maximum(m, s.max(axis=1))
            alpha = np.exp(m - m_new)
            l *= alpha
            acc *= alpha[:, None]
            P = two_o * np.exp(s - m_new[:, None])
            l += P.sum(axis=1)

            def fp4(X):
                # NVFP4 groups of 16 keys start at each key block's first key
                return np.concatenate([nvfp4_along_keys(X[:, cuts[u]:cuts[u + 1]])
                                       for u in range(len(segs))], axis=1)

            if tier == TIER_FULL:
                acc += (P if exact else bf16_rne(P)) @ Vh[keys]
            elif tier == TIER_LOW and low == LOW_FP8:
                acc += (P if exact else e4m3_round(P)) @ qt["dv"][keys]
            elif tier == TIER_LOW:
                acc += (P if exact else fp4(P)) @ qt["dv"][keys]
            else:
                v1, v2 = qt["dv"][keys], qt["rv"][keys]
                if exact:
                    p1, p2 = P, np.zeros_like(P)
                else:
                    p1 = fp4(P)
                    p2 = fp4(fp32_rne(P - p1))
                acc += p1 @ v1 + p1 @ v2 + p2 @ v1
            m = m_new
        pos += cnt
    skips = lst[pos:pos + counts[3]]
    if len(skips):
        s = (q @ rt["kbar_b"][skips].T) * scale
        m_new = np.maximum(m, s.max(axis=1))
        alpha = np.exp(m - m_new)
        l *= alpha
        acc *= alpha[:, None]
        w = rt["n_k"][skips][None, :] * two_o * np.exp(s - m_new[:, None])
        l += w.sum(axis=1)
        acc += (w if exact else bf16_rne(w)) @ rt["vbar_b"][skips]
    return r0, r1, acc / l[:, None]


def tiered_attention_head(Qh, Kh, Vh, rt, qt, low, block_q, block_k, p_offset_log2,
                          scale=0.0, exact=False, qblocks=None, threads=1, key_pack=1):
    """O [N, d] (fp64) of one head; rows of q-blocks not in ``qblocks`` are NaN.
    ``key_pack`` key blocks of one tier share a tile (one running-max update)."""
    N, d = Qh.shape
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    nqb = -(-N // block_q)
    if qblocks is None:
        qblocks = range(nqb)
    O = np.full((N, d), np.nan)
    args = (Qh, Kh, Vh, rt, qt, low, block_q, block_k, p_offset_log2, scale, exact, key_pack)
    if threads > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            results = list(ex.map(lambda i: _qblock(i, *args), qblocks))
    else:
        results = [_qblock(i, *args) for i in qblocks]
    for r0, r1, o in results:
        O[r0:r1] = o
    return O


def tiered_attention(Q, K, V, tau, low, block_q, block_k, p_offset_log2, scale=0.0,
                     keep_diag_full=True, exact=False, heads=None, qblocks=None, threads=1,
                     router=0, price=0.0, kappa=1.0, key_pack=1):
    """Route, quantise and attend over every (b, h) in ``heads`` (default all).

    Q, K, V: fp64 arrays [B, H, N, d] holding bf16 values.  Returns a dict
    {(b, h): {"route": ..., "quant": ..., "O": ...}}."""
    B, H, N, d = Q.shape
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    out = {}
    for b, h in heads:
        rt = route_head(Q[b, h], K[b, h], V[b, h], tau, block_q, block_k, scale, keep_diag_full,
                        router=router, price=price, low=low, kappa=kappa)
        qt = quantize_head(Q[b, h], K[b, h], V[b, h], low, block_q, block_k)
        O = tiered_attention_head(Q[b, h], K[b, h], V[b, h], rt, qt, low, block_q, block_k,
                                  p_offset_log2, rt["scale"], exact, qblocks, threads, key_pack)
        out[(b, h)] = {"route": rt, "quant": qt, "O": O}
    return out


__all__ = ["tiered_attention", "tiered_attention_head", "nvfp4_along_keys",
           "LOW_NONE", "LOW_FP8", "LOW_NVFP4", "LOW_NVFP4_RES"]
