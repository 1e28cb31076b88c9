"""The oracle against the hand-worked cases under ``tests/golden/``.

Each fixture states its inputs, cites the passage its rule follows, and works
every expected value by hand in its comments (no expected value was produced
by running code).  The router rows pin pooling, the n_j-weighted pooled
softmax, the (-M, j) sort with its tie rule, the exclusive prefix against the
thresholds, the forced diagonal and the list order.  The low-tier attention
case pins the power-of-two offset of P', the NVFP4 rounding of P' in groups of
16 keys and of V in groups of 16 tokens per column, and a denominator that
sums P' before rounding; the refine-tier case pins the residual copies (with
e4m3 subnormal scales) and the three-term product that drops A2 B2.  The
price and entropy rows pin the price rule's objectives and spread and the
entropy rule's k = ceil(kappa e^H) with its lift of kept blocks to NVFP4.
The FP8 case pins the power-of-two tile scales and e4m3 rounding; the skip
case pins the n_j weight of a ragged skipped block and the bf16 rounding of
its pseudo-value.
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import route as R
from oracle.attention import tiered_attention
from oracle.quant import LOW_NVFP4, LOW_NVFP4_RES

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read(name):
    """Sections of ``key = value`` lines; a repeated key collects a list."""
    sections, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("[") and line.endswith("]"):
                cur = sections.setdefault(line[1:-1], {})
                continue
            if cur is None:
                cur = sections.setdefault("", {})
            key, _, value = line.partition("=")
            key, value = key.strip(), value.strip()
            if key in cur:
                if not isinstance(cur[key], list):
                    cur[key] = [cur[key]]
                cur[key].append(value)
            else:
                cur[key] = value
    return sections


def _nums(text):
    out = []
    for t in text.split():
        num, _, den = t.partition("/")
        out.append(float(Fraction(num) / Fraction(den or "1")))
    return out


def _ints(text):
    return [int(t) for t in text.split()]


ROUTER = _read("router_rows.txt")


@pytest.mark.parametrize("case", sorted(ROUTER))
def test_router_rows_hand_worked(case):
    sec = ROUTER[case]
    N, block = int(sec["N"]), int(sec["block"])
    w = _nums(sec["w"])
    nkb = -(-N // block)
    assert len(w) == nkb
    Q = np.ones((N, 1))
    K = np.empty((N, 1))
    for j in range(nkb):
        K[j * block:(j + 1) * block] = math.log(w[j])
    rt = R.route_head(Q, K, np.zeros((N, 1)), _nums(sec["tau"]), block, block, scale=1.0)
    mass = np.array(_nums(sec["mass"]))
    flagged = np.array(_ints(sec["flagged"]), dtype=bool)
    rows = sec["row"]
    assert len(rows) == rt["tiers"].shape[0]
    for text in rows:
        head, tiers, counts, lst = [p.strip() for p in text.split("|")]
        i = int(head)
        np.testing.assert_allclose(rt["M"][i], mass, rtol=1e-12)
        np.testing.assert_array_equal(rt["flags"][i], flagged)
        np.testing.assert_array_equal(rt["tiers"][i], _ints(tiers.split(None, 1)[1]))
        np.testing.assert_array_equal(rt["counts"][i], _ints(counts.split(None, 1)[1]))
        np.testing.assert_array_equal(rt["lists"][i], _ints(lst.split(None, 1)[1]))


def _attention_case(name="nvfp4_tier_attention.txt"):
    sec = _read(name)[""]
    N, d, block = int(sec["N"]), int(sec["d"]), int(sec["block"])
    Q = np.zeros((1, 1, N, d))
    K = np.ones((1, 1, N, d))
    V = np.zeros((1, 1, N, d))
    V[0, 0, :4, 0] = 1.0
    V[0, 0, 4:7, 1] = 1.0
    V[0, 0, 7, 1] = 0.75
    return sec, Q, K, V, block


@pytest.mark.parametrize("exact", [False, True])
def test_nvfp4_tier_attention_hand_worked(exact):
    sec, Q, K, V, block = _attention_case()
    out = tiered_attention(Q, K, V, _nums(sec["tau"]), LOW_NVFP4, block, block,
                           int(sec["p_offset_log2"]), exact=exact)[(0, 0)]
    tiers = out["route"]["tiers"]
    np.testing.assert_array_equal(tiers[0], _ints(sec["tiers_qblock0"]))
    np.testing.assert_array_equal(tiers[1], _ints(sec["tiers_qblock1"]))
    O = out["O"]
    tag = "O_exact_qblock" if exact else "O_qblock"
    for qb in range(2):
        want = np.zeros(Q.shape[-1])
        want[:2] = _nums(sec[f"{tag}{qb}"])
        rows = O[qb * block:(qb + 1) * block]
        # dyadic values: the fp64 pass reproduces them up to the rounding of
        # exp(0) - 1 = 0 and of a few exact products, i.e. exactly
        np.testing.assert_allclose(rows, np.broadcast_to(want, rows.shape), rtol=0, atol=1e-15)


def test_nvfp4_residual_tier_attention_hand_worked():
    sec, Q, K, V, block = _attention_case("nvfp4_residual_attention.txt")
    out = tiered_attention(Q, K, V, _nums(sec["tau"]), LOW_NVFP4_RES, block, block,
                           int(sec["p_offset_log2"]))[(0, 0)]
    tiers = out["route"]["tiers"]
    np.testing.assert_array_equal(tiers[0], _ints(sec["tiers_qblock0"]))
    np.testing.assert_array_equal(tiers[1], _ints(sec["tiers_qblock1"]))
    for qb in range(2):
        want = np.zeros(Q.shape[-1])
        want[:2] = _nums(sec[f"O_qblock{qb}"])
        rows = out["O"][qb * block:(qb + 1) * block]
        np.testing.assert_allclose(rows, np.broadcast_to(want, rows.shape), rtol=0, atol=1e-15)


PRICE_ENTROPY = _read("router_price_entropy_rows.txt")


def _check_rows(rt, rows):
    assert len(rows) == rt["tiers"].shape[0]
    for text in rows:
        head, tiers, counts, lst = [p.strip() for p in text.split("|")]
        i = int(head)
        np.testing.assert_array_equal(rt["tiers"][i], _ints(tiers.split(None, 1)[1]))
        np.testing.assert_array_equal(rt["counts"][i], _ints(counts.split(None, 1)[1]))
        np.testing.assert_array_equal(rt["lists"][i], _ints(lst.split(None, 1)[1]))


@pytest.mark.parametrize("case", sorted(PRICE_ENTROPY))
def test_price_and_entropy_router_rows_hand_worked(case):
    sec = PRICE_ENTROPY[case]
    N, block = 320, 64
    w = [8.0, 4.0, 2.0, 1.0, 1.0]
    b = _nums(sec["b"])
    Q = np.ones((N, 1))
    K = np.empty((N, 1))
    for j in range(len(w)):
        rows = np.arange(j * block, (j + 1) * block)
        K[rows, 0] = math.log(w[j]) + np.where(rows % 2 == 0, b[j], -b[j])
    np.testing.assert_allclose(R.block_spread(K, block)[:, 0], np.square(b), rtol=1e-12, atol=1e-15)
    if case.startswith("price"):
        cost = None if sec["cost"] == "default" else _nums(sec["cost"])
        rt = R.route_head(Q, K, np.zeros((N, 1)), (0.5, 0.9), block, block, scale=1.0,
                          router=R.ROUTER_PRICE, price=float(sec["price"]), low=LOW_NVFP4,
                          tier_cost=cost)
        np.testing.assert_allclose(rt["delta"][0], b, rtol=1e-12, atol=1e-15)
    else:
        rt = R.route_head(Q, K, np.zeros((N, 1)), _nums(sec["tau"]), block, block, scale=1.0,
                          router=R.ROUTER_ENTROPY, kappa=float(sec["kappa"]), low=LOW_NVFP4)
        np.testing.assert_array_equal(rt["keep"], int(sec["keep"]))
    np.testing.assert_allclose(rt["M"][0], np.array(w) / 16.0, rtol=1e-12)
    assert not rt["flags"].any()
    _check_rows(rt, sec["row"])


def test_fp8_tier_attention_hand_worked():
    from oracle.quant import LOW_FP8
    sec = _read("fp8_tier_attention.txt")[""]
    N, d, block = int(sec["N"]), int(sec["d"]), int(sec["block"])
    Q = np.zeros((1, 1, N, d))
    K = np.ones((1, 1, N, d))
    V = np.zeros((1, 1, N, d))
    V[0, 0, :4, 0] = 1.0
    V[0, 0, 4:, 1] = float(sec["v_block1"])
    out = tiered_attention(Q, K, V, _nums(sec["tau"]), LOW_FP8, block, block,
                           int(sec["p_offset_log2"]))[(0, 0)]
    tiers = out["route"]["tiers"]
    np.testing.assert_array_equal(tiers[0], _ints(sec["tiers_qblock0"]))
    np.testing.assert_array_equal(tiers[1], _ints(sec["tiers_qblock1"]))
    np.testing.assert_array_equal(out["quant"]["v_scale"], [2.0 ** -8, 2.0 ** -10])
    for qb in range(2):
        want = np.zeros(d)
        want[:2] = _nums(sec[f"O_qblock{qb}"])
        rows = out["O"][qb * block:(qb + 1) * block]
        np.testing.assert_allclose(rows, np.broadcast_to(want, rows.shape), rtol=0, atol=1e-15)


def test_skip_tier_attention_hand_worked():
    from oracle.quant import LOW_FP8
    sec = _read("skip_tier_attention.txt")[""]
    N, d, block = int(sec["N"]), int(sec["d"]), int(sec["block"])
    Q = np.zeros((1, 1, N, d))
    K = np.ones((1, 1, N, d))
    V = np.zeros((1, 1, N, d))
    V[0, 0, :4, 0] = 1.0
    V[0, 0, 4:6, 1] = 1.0
    V[0, 0, 6, 1] = 0.75
    out = tiered_attention(Q, K, V, _nums(sec["tau"]), LOW_FP8, block, block,
                           int(sec["p_offset_log2"]))[(0, 0)]
    tiers = out["route"]["tiers"]
    np.testing.assert_array_equal(tiers[0], _ints(sec["tiers_qblock0"]))
    np.testing.assert_array_equal(tiers[1], _ints(sec["tiers_qblock1"]))
    for qb in range(2):
        want = np.zeros(d)
        want[:2] = _nums(sec[f"O_qblock{qb}"])
        rows = out["O"][qb * block:min(N, (qb + 1) * block)]
        np.testing.assert_allclose(rows, np.broadcast_to(want, rows.shape), rtol=1e-15, atol=1e-15)
