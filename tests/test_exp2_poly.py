"""The exponential the attention kernel runs on the FMA pipe for a share of
each row's P' (exp2_poly2 in ta_attn_common.cuh), replayed step by step in
fp32 on the CPU with the coefficients read from that header: its relative
error against 2^x must stay below 1.1e-4 (the minimax fit's bound) over the
whole argument range the softmax produces, integer arguments must give exact
powers of two, and masked columns (-inf) must come out negligible."""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "precision_attention_video_b200", "csrc", "ta_attn_common.cuh")


def _coeffs():
    src = open(HDR).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(x) for x in re.findall(r"pack2\(([0-9.eE+-]+)f, \1f\)", body)]
    # order of appearance: c3, c2, c1, then the constant 1
    c3, c2, c1, c0 = vals[-4:]
    assert c0 == 1.0
    return np.float32(c1), np.float32(c2), np.float32(c3)


def _fma(a, b, c):
    """fp32 fused multiply-add: the product is exact in fp64, one rounding."""
    return np.float32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def exp2_poly(a):
    c1, c2, c3 = _coeffs()
    a = np.asarray(a, dtype=np.float32)
    x = np.maximum(a, np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = np.float32(x + magic)
    j = np.float32(t - magic)
    f = _fma(j, np.float32(-1.0), x)
    p = _fma(f, c3, np.full_like(f, c2))
    p = _fma(f, p, np.full_like(f, c1))
    p = _fma(f, p, np.full_like(f, np.float32(1.0)))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        np.linspace(-0.5, 0.5, 200001, dtype=np.float32),          # every reduced argument
        rng.uniform(-120.0, 15.0, 500000).astype(np.float32),       # P' = 2^(o + (s - m) c2)
        np.float32(np.arange(-100, 16)) + np.float32(0.5),          # rounding ties of rint
    ])
    y = exp2_poly(xs).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 1.1e-4, rel.max()


def test_integer_arguments_are_exact_powers_of_two():
    k = np.arange(-124, 16, dtype=np.float32)
    np.testing.assert_array_equal(exp2_poly(k), np.exp2(k.astype(np.float64)).astype(np.float32))


def test_masked_columns_come_out_negligible():
    y = exp2_poly(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -124)
