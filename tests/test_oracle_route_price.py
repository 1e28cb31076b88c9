"""Pins of the oracle's price router (Triage's single-price tier rule, as
oracle/route.py states it): closed forms of the block spread, skip exactness
on blocks of equal keys against dense attention, the price limits, the
monotone response to the price, and the abstract's own wording of the rule
(no tile could move to a more accurate tier for an error reduction worth its
extra compute, nor to a cheaper one without losing more than it saves)."""

import numpy as np
import pytest

import oracle
from oracle import formats as F
from oracle import quant as Qz
from oracle import route as R
from oracle.attention import tiered_attention_head

RANK = {R.TIER_SKIP: 0, R.TIER_LOW: 1, R.TIER_RES: 2, R.TIER_FULL: 3}


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_block_spread_closed_form():
    # rows base + a u and base - a u alternate: mean base, variance a^2 along
    # u's coordinate and 0 along every other
    rng = np.random.default_rng(3)
    d, blk, a = 16, 8, 0.75
    u = np.zeros(d)
    u[5] = 1.0
    base = rng.normal(size=(3, d))
    X = np.concatenate([np.stack([b + (a if r % 2 == 0 else -a) * u for r in range(blk)]) for b in base])
    var = R.block_spread(X, blk)
    assert var.shape == (3, d)
    assert np.allclose(var[:, 5], a * a, rtol=0, atol=1e-15)
    assert np.allclose(np.delete(var, 5, axis=1), 0.0, rtol=0, atol=1e-15)
    # a ragged tail block of one row has no spread
    assert (R.block_spread(np.concatenate([X, base[:1]]), blk)[-1] == 0.0).all()


def test_delta_is_the_rms_logit_spread_when_key_coordinates_are_independent():
    # keys with independent +-a_c signs per coordinate (all 2^d patterns): for
    # each query q the variance of q . k over the block is exactly
    # sum_c q_c^2 a_c^2, so the mean over the block's queries is
    # sum_c (qbar_c^2 + qvar_c) a_c^2, the router's delta^2 / scale^2
    rng = np.random.default_rng(9)
    d, blk = 8, 256
    a = rng.uniform(0.1, 1.0, size=d)
    signs = np.array([[1 if (r >> c) & 1 else -1 for c in range(d)] for r in range(blk)])
    Kb = signs * a
    Q = rng.normal(size=(blk, d)) + 0.5
    rt = R.route_head(Q, Kb, Kb, None, blk, blk, router=R.ROUTER_PRICE, price=0.0,
                      low=Qz.LOW_NVFP4, keep_diag_full=False)
    per_query_var = ((Q @ Kb.T) * rt["scale"]).var(axis=1)
    want = np.sqrt(per_query_var.mean())
    assert abs(rt["delta"][0, 0] - want) <= 1e-12 * want


def _blocky(N, d, bk, seed):
    """Q random; K and V constant inside each key block (bf16 values)."""
    rng = np.random.default_rng(seed)
    Q = F.bf16_rne(rng.normal(size=(N, d)) * 2)
    nkb = -(-N // bk)
    Kb = F.bf16_rne(rng.normal(size=(nkb, d)) * 2)
    Vb = F.bf16_rne(rng.normal(size=(nkb, d)))
    K = np.repeat(Kb, bk, axis=0)[:N]
    V = np.repeat(Vb, bk, axis=0)[:N]
    return Q, K, V


@pytest.mark.parametrize("N,bq,bk,d", [(320, 64, 64, 32), (300, 128, 64, 16)])
@pytest.mark.parametrize("price", [0.0, 1e-4, 1.0])
def test_equal_keys_are_skipped_and_skip_is_exact(N, bq, bk, d, price):
    Q, K, V = _blocky(N, d, bk, seed=N + d)
    low = Qz.LOW_NVFP4_RES
    rt = R.route_head(Q, K, V, None, bq, bk, router=R.ROUTER_PRICE, price=price, low=low)
    assert (rt["kvar"] == 0.0).all() and (rt["delta"] == 0.0).all()
    for i in range(rt["tiers"].shape[0]):
        diag = set(R.diag_blocks(i, bq, bk, N))
        for j in range(rt["tiers"].shape[1]):
            assert rt["tiers"][i, j] == (R.TIER_FULL if j in diag else R.TIER_SKIP)
    qt = Qz.quantize_head(Q, K, V, low, bq, bk)
    O = tiered_attention_head(Q, K, V, rt, qt, low, bq, bk, 11, rt["scale"], exact=True)
    assert _rel(O, oracle.dense_attention(Q, K, V)) <= 1e-12


def _random(N, d, seed):
    rng = np.random.default_rng(seed)
    return [F.bf16_rne(rng.normal(size=(N, d)) * s) for s in (2.0, 2.0, 1.0)]


@pytest.mark.parametrize("low", [Qz.LOW_NONE, Qz.LOW_FP8, Qz.LOW_NVFP4, Qz.LOW_NVFP4_RES])
def test_price_limits(low):
    Q, K, V = _random(512, 32, seed=low)
    rt0 = R.route_head(Q, K, V, None, 64, 64, router=R.ROUTER_PRICE, price=0.0, low=low)
    assert rt0["delta"].min() > 2.0 ** -8
    assert (rt0["tiers"] == R.TIER_FULL).all()
    rtx = R.route_head(Q, K, V, None, 64, 64, router=R.ROUTER_PRICE, price=1e30, low=low)
    for i in range(rtx["tiers"].shape[0]):
        diag = set(R.diag_blocks(i, 64, 64, 512))
        for j in range(rtx["tiers"].shape[1]):
            assert rtx["tiers"][i, j] == (R.TIER_FULL if j in diag else R.TIER_SKIP)


def test_tiers_fall_monotonically_with_price():
    Q, K, V = _random(640, 32, seed=11)
    prev = None
    for price in [0.0, 1e-6, 1e-5, 3e-5, 1e-4, 3e-4, 1e-3, 1e-2, 1.0]:
        rt = R.route_head(Q, K, V, None, 64, 64, router=R.ROUTER_PRICE, price=price,
                          low=Qz.LOW_NVFP4_RES, keep_diag_full=False)
        rank = np.vectorize(RANK.get)(rt["tiers"])
        if prev is not None:
            assert (rank <= prev).all()
        prev = rank
    assert prev.max() == 0


@pytest.mark.parametrize("tier_cost,n_tiers,prices", [
    # nominal tensor-pipe rates: every tier has a use
    ((0.0, 1.0, 3.0, 4.0), 3, (3e-3, 1e-2, 2e-2, 3e-2)),
    # the defaults (measured kernel time): NVFP4 and the residual tier cost
    # more than bf16, only skip and full pay
    (None, 2, (3e-2, 0.1, 0.3, 1.0)),
])
def test_no_move_pays_at_the_price(tier_cost, n_tiers, prices):
    Q, K, V = _random(640, 32, seed=5)
    low = Qz.LOW_NVFP4_RES
    table = R.price_tiers(low, tier_cost)
    cost = [c for _, _, c in table]
    seen = set()
    for price in prices:
        rt = R.route_head(Q, K, V, None, 64, 64, router=R.ROUTER_PRICE, price=price, low=low,
                          keep_diag_full=False, tier_cost=tier_cost)
        M, delta, tiers = rt["M"], rt["delta"], rt["tiers"]
        for i in range(M.shape[0]):
            for j in range(M.shape[1]):
                k = [t for t, _, _ in table].index(tiers[i, j])
                seen.add(int(tiers[i, j]))
                err = [M[i, j] * (delta[i, j] if eps is None else eps) for _, eps, _ in table]
                for t in range(len(table)):
                    if cost[t] > cost[k]:    # more accurate: the error it saves is not worth the compute
                        assert err[k] - err[t] <= price * (cost[t] - cost[k]) * (1 + 1e-12)
                    elif cost[t] < cost[k]:  # cheaper: it would lose more error than the compute it saves
                        assert err[t] - err[k] > price * (cost[k] - cost[t]) * (1 - 1e-12)
    assert len(seen) >= n_tiers   # the prices above spread tiles over several tiers
