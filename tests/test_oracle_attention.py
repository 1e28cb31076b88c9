"""Pins of the oracle's tiered attention against closed forms.

* all tiles full, exact mode -> naive fp64 softmax attention;
* every key block constant, all off-diagonal tiles skipped, exact mode -> dense
  attention (block j of n_j equal keys contributes n_j exp(q.k_j) v_j exactly,
  the skip formula of "Triage", zhuanzhiai paper page, abstract);
* operands already on the FP8 / NVFP4 grid, exact mode -> low tier = dense;
* two-level NVFP4 operands (x = deq1 + deq2 exactly), exact mode -> the refine
  tier's logits are (Q K^T - R_Q R_K^T) * scale (the dropped second-order term);
* the power-of-two offset 2^o cancels;
* the non-exact full tier differs from dense only by bf16 rounding of P'.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import formats as F
from oracle import quant as Qz
from oracle import route as R
from oracle.attention import tiered_attention_head


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _run(Q, K, V, tau, low, bq, bk, o=8, exact=True, keep_diag=True):
    rt = R.route_head(Q, K, V, tau, bq, bk, keep_diag_full=keep_diag)
    qt = Qz.quantize_head(Q, K, V, low, bq, bk)
    return tiered_attention_head(Q, K, V, rt, qt, low, bq, bk, o, rt["scale"], exact), rt


@pytest.mark.parametrize("N,bq,bk,d", [(200, 64, 64, 32), (256, 128, 64, 64), (300, 64, 128, 16),
                                    (300, 128, 32, 16)])
def test_all_full_equals_dense(N, bq, bk, d):
    rng = np.random.default_rng(N)
    Q, K, V = (F.bf16_rne(rng.normal(size=(N, d)) * 2) for _ in range(3))
    O, rt = _run(Q, K, V, (2.0, 2.0), Qz.LOW_FP8, bq, bk)
    assert (rt["tiers"] == R.TIER_FULL).all()
    D = oracle.dense_attention(Q, K, V)
    assert _rel(O, D) <= 1e-12
    # non-exact: P' rounded to bf16 before PV; error at the bf16 level only
    O2, _ = _run(Q, K, V, (2.0, 2.0), Qz.LOW_FP8, bq, bk, exact=False)
    e = _rel(O2, D)
    assert 1e-5 < e < 8e-3


def test_skip_exact_on_constant_blocks():
    rng = np.random.default_rng(7)
    N, bk, d = 320, 64, 32
    nb = N // bk
    kb = F.bf16_rne(rng.normal(size=(nb, d)))
    vb = F.bf16_rne(rng.normal(size=(nb, d)))
    K = np.repeat(kb, bk, axis=0)
    V = np.repeat(vb, bk, axis=0)
    Q = F.bf16_rne(rng.normal(size=(N, d)))
    O, rt = _run(Q, K, V, (0.0, 0.0), Qz.LOW_FP8, 64, bk)
    # only the diagonal is kept
    for i in range(nb):
        assert rt["tiers"][i, i] == R.TIER_FULL
        assert (np.delete(rt["tiers"][i], i) == R.TIER_SKIP).all()
    D = oracle.dense_attention(Q, K, V)
    assert _rel(O, D) <= 1e-12


def test_skip_weights_ragged_block():
    # a ragged tail block of 8 equal keys must weigh 8x one key
    rng = np.random.default_rng(8)
    N, d = 72, 16
    K = np.zeros((N, d))
    V = np.zeros((N, d))
    K[:64] = F.bf16_rne(rng.normal(size=d))
    K[64:] = F.bf16_rne(rng.normal(size=d))
    V[:64] = F.bf16_rne(rng.normal(size=d))
    V[64:] = F.bf16_rne(rng.normal(size=d))
    Q = F.bf16_rne(rng.normal(size=(N, d)))
    O, rt = _run(Q, K, V, (0.0, 0.0), Qz.LOW_FP8, 64, 64)
    assert rt["tiers"][0, 1] == R.TIER_SKIP and rt["tiers"][1, 0] == R.TIER_SKIP
    assert _rel(O, oracle.dense_attention(Q, K, V)) <= 1e-12


def test_fp8_low_grid_exact_equals_dense():
    rng = np.random.default_rng(9)
    N, d = 256, 32

    def grid():
        c = rng.integers(0x20, 0x60, size=(N, d)).astype(np.uint8) | (rng.integers(0, 2, (N, d)) << 7).astype(np.uint8)
        X = F.e4m3_decode(c) / 64.0            # tile amax in (3.5, 7] -> scale 2^-6, exact
        X[::64, 0] = 7.0
        return X

    Q, K, V = grid(), grid(), grid()
    O, rt = _run(Q, K, V, (0.0, 2.0), Qz.LOW_FP8, 64, 64, keep_diag=False)
    assert (rt["tiers"] == R.TIER_LOW).all()
    assert _rel(O, oracle.dense_attention(Q, K, V)) <= 1e-12
    # non-exact: P' rounded to e4m3 before PV: error near the e4m3 level
    O2, _ = _run(Q, K, V, (0.0, 2.0), Qz.LOW_FP8, 64, 64, keep_diag=False, exact=False)
    assert 1e-4 < _rel(O2, oracle.dense_attention(Q, K, V)) < 5e-2


def _nvfp4_grid_rows(rng, N, d):
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    X = vals[rng.integers(0, 8, (N, d))] * rng.choice([-1.0, 1.0], (N, d))
    X[:, ::16] = 6.0
    return X * 2.0 ** rng.integers(-3, 1, (N, d // 16)).repeat(16, axis=1)


def test_nvfp4_low_grid_exact_equals_dense():
    rng = np.random.default_rng(10)
    N, d = 256, 32
    Q, K = _nvfp4_grid_rows(rng, N, d), _nvfp4_grid_rows(rng, N, d)
    V = _nvfp4_grid_rows(rng, d, N).T.copy()   # groups of 16 tokens per column
    O, rt = _run(Q, K, V, (0.0, 2.0), Qz.LOW_NVFP4, 128, 128, o=11, keep_diag=False)
    assert (rt["tiers"] == R.TIER_LOW).all()
    assert _rel(O, oracle.dense_attention(Q, K, V)) <= 1e-12


def test_residual_tier_drops_only_second_order_term():
    rng = np.random.default_rng(11)
    N, d = 256, 32
    # x = A + Rr: A on the NVFP4 grid with scale 1 (group amax 6), Rr on the
    # grid with scale 2^-5 and |Rr| <= 0.1875 < half a quantum of A, so that
    # deq1(x) = A and the residual copy is exactly Rr.
    def two_level(n, dd):
        vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
        A = vals[rng.integers(0, 8, (n, dd))] * rng.choice([-1.0, 1.0], (n, dd))
        A[:, ::16] = 6.0
        Rr = vals[rng.integers(0, 8, (n, dd))] * rng.choice([-1.0, 1.0], (n, dd)) / 32.0
        Rr[:, ::16] = 6.0 / 32.0
        return A + Rr, Rr

    Q, RQ = two_level(N, d)
    K, RK = two_level(N, d)
    Vt, _ = two_level(d, N)
    V = Vt.T.copy()
    rt = R.route_head(Q, K, V, (0.0, 2.0, 2.0), 128, 128, keep_diag_full=False)
    qt = Qz.quantize_head(Q, K, V, Qz.LOW_NVFP4_RES, 128, 128)
    np.testing.assert_array_equal(qt["rq"], RQ)
    np.testing.assert_array_equal(qt["rk"], RK)
    assert (rt["tiers"] == R.TIER_RES).all()
    O = tiered_attention_head(Q, K, V, rt, qt, Qz.LOW_NVFP4_RES, 128, 128, 11, rt["scale"], True)
    s = (Q @ K.T - RQ @ RK.T) / math.sqrt(d)
    p = np.exp(s - s.max(1, keepdims=True))
    want = (p @ V) / p.sum(1, keepdims=True)
    assert _rel(O, want) <= 1e-12


def test_offset_cancels():
    rng = np.random.default_rng(12)
    N, d = 192, 32
    Q, K, V = (F.bf16_rne(rng.normal(size=(N, d)) * 2) for _ in range(3))
    a, _ = _run(Q, K, V, (0.5, 0.8), Qz.LOW_FP8, 64, 64, o=0)
    b, _ = _run(Q, K, V, (0.5, 0.8), Qz.LOW_FP8, 64, 64, o=8)
    assert _rel(a, b) <= 1e-13


def test_tiers_mix_reasonable_on_generator_input():
    from latent_gen import get_config, make_qkv
    import torch
    cfg = get_config("tiny")
    Q, K, V = (x.to(torch.float64).numpy() for x in make_qkv(cfg))
    res = oracle.tiered_attention(Q, K, V, cfg.tau, cfg.low, cfg.block_q, cfg.block_k,
                                  cfg.p_offset_log2, heads=[(0, 1)])
    r = res[(0, 1)]
    t = r["route"]["tiers"]
    assert (t == R.TIER_FULL).any() and (t == R.TIER_LOW).any() and (t == R.TIER_SKIP).any()
    D = oracle.dense_attention(Q[0, 1], K[0, 1], V[0, 1])
    assert _rel(r["O"], D) < 0.3          # an approximation, but not garbage


def test_fine_grained_key_blocks_of_32():
    # FG-Attn ("FG-Attn" searcharxiv author page, abstract) skips at M x N
    # granularity with M >= 16, N >= 1; the tiered method at N = 32 keys and
    # M = 128 queries is the same pass over 32-key blocks.  Three exact cases:
    rng = np.random.default_rng(12)
    N, d, bq, bk = 296, 32, 128, 32               # 9 full key blocks and an 8-key tail
    # (1) constant 32-key blocks: skipping them is exact
    nb = -(-N // bk)
    K = np.repeat(F.bf16_rne(rng.normal(size=(nb, d))), bk, axis=0)[:N]
    V = np.repeat(F.bf16_rne(rng.normal(size=(nb, d))), bk, axis=0)[:N]
    Q = F.bf16_rne(rng.normal(size=(N, d)))
    O, rt = _run(Q, K, V, (0.0, 0.0), Qz.LOW_FP8, bq, bk)
    assert (rt["tiers"] == R.TIER_SKIP).sum() > 0
    assert rt["n_k"][-1] == N - (nb - 1) * bk
    assert _rel(O, oracle.dense_attention(Q, K, V)) <= 1e-12
    # (2) operands on the NVFP4 grid, every tile low: a 32-key tile holds two
    # whole 16-token V groups and two 16-key P groups, so exact=True is dense
    N2 = 256
    Q2, K2 = _nvfp4_grid_rows(rng, N2, d), _nvfp4_grid_rows(rng, N2, d)
    V2 = _nvfp4_grid_rows(rng, d, N2).T.copy()
    O2, rt2 = _run(Q2, K2, V2, (0.0, 2.0), Qz.LOW_NVFP4, bq, bk, o=11, keep_diag=False)
    assert (rt2["tiers"] == R.TIER_LOW).all()
    assert _rel(O2, oracle.dense_attention(Q2, K2, V2)) <= 1e-12
    # (3) the diagonal of a 128-row query block covers four 32-key blocks
    assert R.diag_blocks(1, bq, bk, N) == [4, 5, 6, 7]
    assert all((rt["tiers"][1, 4:8] == R.TIER_FULL))


def _expand_plan(rt, sub, nb_sub):
    """The plan of 128-key blocks rewritten over key blocks `sub` times
    narrower: block j becomes blocks sub*j .. sub*j + sub - 1, same tier,
    same list position."""
    counts = rt["counts"] * 0
    lists = []
    for i in range(len(rt["counts"])):
        row, pos = [], 0
        for t in range(4):
            c = int(rt["counts"][i][t])
            blocks = [sub * j + u for j in rt["lists"][i][pos:pos + c] for u in range(sub)
                      if sub * j + u < nb_sub]
            counts[i][t] = len(blocks)
            row += blocks
            pos += c
        lists.append(row)
    return {"counts": counts, "lists": np.array(lists, dtype=np.int32), "n_k": None}


@pytest.mark.parametrize("low,tau", [(Qz.LOW_NVFP4, (0.5, 2.0)), (Qz.LOW_NVFP4_RES, (0.3, 0.6, 2.0))])
def test_key_pack_of_narrow_blocks_equals_one_wide_block(low, tau):
    # A tile that packs the four 32-key blocks of one 128-key block computes
    # what the 128-key tile does: the same keys, one running-max update, P'
    # groups of 16 keys from the same starts.  Rounded P', ragged 24-key tail.
    rng = np.random.default_rng(21)
    N, d, bq = 376, 32, 128
    Q, K, V = (F.bf16_rne(rng.normal(size=(N, d)) * 2) for _ in range(3))
    rt = R.route_head(Q, K, V, tau, bq, 128)
    assert (rt["tiers"] != R.TIER_SKIP).all() and (rt["tiers"] != R.TIER_FULL).any()
    qt = Qz.quantize_head(Q, K, V, low, bq, 128)
    qt32 = Qz.quantize_head(Q, K, V, low, bq, 32)
    for key in ("dq", "dk", "dv"):
        np.testing.assert_array_equal(qt[key], qt32[key])
    wide = tiered_attention_head(Q, K, V, rt, qt, low, bq, 128, 11, rt["scale"], False)
    rt32 = _expand_plan(rt, 4, -(-N // 32))
    narrow = tiered_attention_head(Q, K, V, rt32, qt32, low, bq, 32, 11, rt["scale"], False,
                                   key_pack=4)
    one_by_one = tiered_attention_head(Q, K, V, rt32, qt32, low, bq, 32, 11, rt["scale"], False)
    assert _rel(narrow, wide) <= 1e-12
    assert _rel(one_by_one, wide) > 1e-6      # the grouping is what makes them equal


def test_key_pack_order_inside_a_tile_is_immaterial():
    # Within one packed tile the order of its key blocks changes neither the
    # running maximum nor any P' group (groups start at each block's first
    # key), so reversing every pack changes only summation order -- also when
    # the ragged 24-key block moves from the end of a pack to its front.
    rng = np.random.default_rng(22)
    N, d, bq, bk = 376, 32, 128, 32
    Q, K, V = (F.bf16_rne(rng.normal(size=(N, d)) * 2) for _ in range(3))
    low = Qz.LOW_NVFP4
    rt = R.route_head(Q, K, V, (0.3, 2.0), bq, bk)
    qt = Qz.quantize_head(Q, K, V, low, bq, bk)
    rev = dict(rt)
    lists = rt["lists"].copy()
    moved = False
    for i in range(len(lists)):
        pos = 0
        for t in range(3):
            c = int(rt["counts"][i][t])
            for g0 in range(pos, pos + c, 4):
                g1 = min(pos + c, g0 + 4)
                if g1 - g0 > 1 and lists[i][g1 - 1] == 11:
                    moved = True
                lists[i][g0:g1] = lists[i][g0:g1][::-1].copy()
            pos += c
    rev["lists"] = lists
    assert moved
    a = tiered_attention_head(Q, K, V, rt, qt, low, bq, bk, 11, rt["scale"], False, key_pack=4)
    b = tiered_attention_head(Q, K, V, rev, qt, low, bq, bk, 11, rt["scale"], False, key_pack=4)
    assert _rel(a, b) <= 1e-12
