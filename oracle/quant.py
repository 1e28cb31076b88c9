"""Low-precision copies of Q, K, V for the low and refine tiers (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

"Triage" (zhuanzhiai paper page, abstract) skims tiles in NVFP4 and refines
them with an NVFP4 residual correction; the FP8 e4m3 low tier is the other
reduced precision the workloads name.  The pages fix no scaling rule, so:

* FP8 e4m3, one scale per tile of rows (Bq rows of Q, Bk rows of K or V), over
  the tile's real rows only.  Reading: the scale is the smallest power of two
  s with amax <= 448 s (s = 1 when amax = 0), i.e. 2^ceil(log2(amax/448)); a
  power of two keeps x/s exact and lets the scale be applied exactly later.
  code = e4m3_RNE_satfinite(x / s); dequantised value = e4m3(code) * s.
* NVFP4, one ue4m3 scale per 16 consecutive elements: along d for rows of Q
  and K, along tokens (aligned to token 0, zero padding past N) for each column
  of V, so that the PV product's reduction runs over 16-element groups.
  sc = ue4m3_RNE_satfinite(fp32(amax / 6)); if sc = 0 every code is 0;
  otherwise inv = fp32(1 / sc) and code = e2m1_RNE_satfinite(fp32(x * inv));
  dequantised value = e2m1(code) * sc.  Reading: a single scale level, rounded
  to nearest (so x * inv may exceed 6 and saturate).
* Residual: r = fp32(x - dequant(x)), then NVFP4 of r with its own scales.
"""

from __future__ import annotations

import math

import numpy as np

from .formats import (e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, fp32_rne,
                      ue4m3_decode, ue4m3_encode)

LOW_NONE, LOW_FP8, LOW_NVFP4, LOW_NVFP4_RES = 0, 1, 2, 3


def fp8_tile_scale(amax: float) -> float:
    """Smallest power of two s with amax <= 448 * s; 1 when amax is 0."""
    amax = float(amax)
    if amax == 0.0:
        return 1.0
    m, e = math.frexp(amax)          # amax = m * 2^e, 0.5 <= m < 1; 448 = 0.875 * 2^9
    k = e - 9 if m <= 0.875 else e - 8
    return math.ldexp(1.0, k)


def quant_fp8_tiles(X: np.ndarray, block: int):
    """FP8 codes [N, d] and per-tile scales [ceil(N/block)] of rows of X."""
    N = X.shape[0]
    nb = -(-N // block)
    codes = np.empty(X.shape, dtype=np.uint8)
    scales = np.empty(nb, dtype=np.float64)
    for b in range(nb):
        rows = slice(b * block, min(N, (b + 1) * block))
        s = fp8_tile_scale(np.max(np.abs(X[rows])) if X[rows].size else 0.0)
        scales[b] = s
        codes[rows] = e4m3_encode(X[rows] / s)
    return codes, scales


def dequant_fp8_tiles(codes: np.ndarray, scales: np.ndarray, block: int) -> np.ndarray:
    out = e4m3_decode(codes)
    for b, s in enumerate(scales):
        out[b * block:(b + 1) * block] *= s
    return out


def nvfp4_quant_groups(G: np.ndarray):
    """NVFP4 of groups along the last axis (length 16): (codes, scale codes)."""
    G = np.asarray(G, dtype=np.float64)
    amax = np.max(np.abs(G), axis=-1)
    sc_code = ue4m3_encode(fp32_rne(amax / 6.0))
    sc = ue4m3_decode(sc_code)
    nz = sc > 0
    inv = np.where(nz, fp32_rne(1.0 / np.where(nz, sc, 1.0)), 0.0)
    y = fp32_rne(G * inv[..., None])
    codes = np.where(nz[..., None], e2m1_encode(y), np.uint8(0)).astype(np.uint8)
    return codes, sc_code


def nvfp4_dequant_groups(codes: np.ndarray, sc_code: np.ndarray) -> np.ndarray:
    return e2m1_decode(codes) * ue4m3_decode(sc_code)[..., None]


def quant_nvfp4_rows(X: np.ndarray):
    """NVFP4 with groups of 16 along the last axis: codes [N, d], scales [N, d/16]."""
    N, d = X.shape
    codes, sc = nvfp4_quant_groups(X.reshape(N, d // 16, 16))
    return codes.reshape(N, d), sc


def dequant_nvfp4_rows(codes: np.ndarray, sc: np.ndarray) -> np.ndarray:
    N, d = codes.shape
    return nvfp4_dequant_groups(codes.reshape(N, d // 16, 16), sc).reshape(N, d)


def quant_nvfp4_cols(X: np.ndarray):
    """NVFP4 with groups of 16 consecutive rows per column (aligned to row 0,
    zero padding past N): codes [Np, d] and scales [Np/16, d], Np = 16*ceil(N/16)."""
    N, d = X.shape
    Np = -(-N // 16) * 16
    Xp = np.zeros((Np, d))
    Xp[:N] = X
    G = Xp.reshape(Np // 16, 16, d).transpose(0, 2, 1)          # [g, d, 16]
    codes, sc = nvfp4_quant_groups(G)
    return codes.transpose(0, 2, 1).reshape(Np, d), sc


def dequant_nvfp4_cols(codes: np.ndarray, sc: np.ndarray) -> np.ndarray:
    Np, d = codes.shape
    G = codes.reshape(Np // 16, 16, d).transpose(0, 2, 1)
    return nvfp4_dequant_groups(G, sc).transpose(0, 2, 1).reshape(Np, d)


def quantize_head(Qh, Kh, Vh, low: int, block_q: int, block_k: int) -> dict:
    """All low-precision copies of one head's Q, K, V (fp64 values of bf16).

    Returns a dict with codes, scales and dequantised values ("dq", "dk", "dv";
    "rq", "rk", "rv" hold the dequantised residual copies for LOW_NVFP4_RES).
    dv has Np rows for NVFP4 (zero padding past N)."""
    out = {"low": low}
    if low == LOW_NONE:
        return out
    if low == LOW_FP8:
        out["q_codes"], out["q_scale"] = quant_fp8_tiles(Qh, block_q)
        out["k_codes"], out["k_scale"] = quant_fp8_tiles(Kh, block_k)
        out["v_codes"], out["v_scale"] = quant_fp8_tiles(Vh, block_k)
        out["dq"] = dequant_fp8_tiles(out["q_codes"], out["q_scale"], block_q)
        out["dk"] = dequant_fp8_tiles(out["k_codes"], out["k_scale"], block_k)
        out["dv"] = dequant_fp8_tiles(out["v_codes"], out["v_scale"], block_k)
        return out
    if low not in (LOW_NVFP4, LOW_NVFP4_RES):
        raise ValueError(f"unknown low format {low}")
    out["q_codes"], out["q_sc"] = quant_nvfp4_rows(Qh)
    out["k_codes"], out["k_sc"] = quant_nvfp4_rows(Kh)
    out["v_codes"], out["v_sc"] = quant_nvfp4_cols(Vh)
    out["dq"] = dequant_nvfp4_rows(out["q_codes"], out["q_sc"])
    out["dk"] = dequant_nvfp4_rows(out["k_codes"], out["k_sc"])
    out["dv"] = dequant_nvfp4_cols(out["v_codes"], out["v_sc"])
    if low == LOW_NVFP4_RES:
        N = Vh.shape[0]
        rq = fp32_rne(Qh - out["dq"])
        rk = fp32_rne(Kh - out["dk"])
        rv = fp32_rne(Vh - out["dv"][:N])
        out["rq_codes"], out["rq_sc"] = quant_nvfp4_rows(rq)
        out["rk_codes"], out["rk_sc"] = quant_nvfp4_rows(rk)
        out["rv_codes"], out["rv_sc"] = quant_nvfp4_cols(rv)
        out["rq"] = dequant_nvfp4_rows(out["rq_codes"], out["rq_sc"])
        out["rk"] = dequant_nvfp4_rows(out["rk_codes"], out["rk_sc"])
        out["rv"] = dequant_nvfp4_cols(out["rv_codes"], out["rv_sc"])
    return out
