"""Pins of the oracle's entropy router (HierPAS's entropy-derived retention,
as oracle/route.py states it): the row's kept-block count against the closed
forms of uniform and one-hot pooled distributions, the kept set being the
heaviest blocks, precision inside it by the prefix rule, and the retention
scale's limits."""

import math

import numpy as np
import pytest

from oracle import formats as F
from oracle import route as R

RANK = {R.TIER_SKIP: 0, R.TIER_LOW: 1, R.TIER_RES: 2, R.TIER_FULL: 3}


def test_uniform_row_keeps_every_block():
    # H = ln n, so exp(H) = n effective blocks: all kept (kappa = 1)
    n = 12
    M = np.full(n, 1.0 / n)
    tiers, flags, k = R.assign_tiers_entropy(M, (0.5, 0.9), 1.0)
    assert k == n and (tiers != R.TIER_SKIP).all()
    # exp(ln 12) sits on an integer: the row is flagged
    assert flags.all()


def test_one_hot_row_keeps_one_block():
    M = np.zeros(9)
    M[4] = 1.0
    tiers, _, k = R.assign_tiers_entropy(M, (0.5, 0.9), 1.0)
    assert k == 1
    assert tiers[4] == R.TIER_FULL and (np.delete(tiers, 4) == R.TIER_SKIP).all()


def test_two_level_row_closed_form():
    # m blocks of mass a and the rest of mass b: H in closed form
    n, m = 20, 5
    a = 0.15
    b = (1.0 - m * a) / (n - m)
    M = np.array([a] * m + [b] * (n - m))
    H = -(m * a * math.log(a) + (n - m) * b * math.log(b))
    for kappa in (0.3, 0.5, 1.0):
        _, _, k = R.assign_tiers_entropy(M, (0.3, 0.95), kappa)
        assert k == min(n, max(1, math.ceil(kappa * math.exp(H))))


@pytest.mark.parametrize("kappa", [0.05, 0.3, 0.7, 1.0, 3.0])
def test_kept_set_is_heaviest_and_precision_follows_the_prefix(kappa):
    rng = np.random.default_rng(7)
    M = rng.exponential(size=40) ** 3
    M /= M.sum()
    tau = (0.5, 0.8)
    tiers, _, k = R.assign_tiers_entropy(M, tau, kappa)
    base, _ = R.assign_tiers(M, tau)
    order = np.lexsort((np.arange(40), -M))
    kept = set(order[:k].tolist())
    for r, j in enumerate(order):
        if j in kept:
            assert tiers[j] != R.TIER_SKIP
            want = base[j] if base[j] != R.TIER_SKIP else R.TIER_LOW
            assert tiers[j] == want
        else:
            assert tiers[j] == R.TIER_SKIP
    # a larger retention scale never keeps less precision anywhere
    t2, _, k2 = R.assign_tiers_entropy(M, tau, kappa * 2)
    assert k2 >= k
    assert all(RANK[t2[j]] >= RANK[tiers[j]] for j in range(40))


def test_route_head_entropy_diagonal_and_keep_counts():
    rng = np.random.default_rng(1)
    N, d = 640, 32
    Q, K, V = (F.bf16_rne(rng.normal(size=(N, d)) * s) for s in (3.0, 3.0, 1.0))
    rt = R.route_head(Q, K, V, (0.6, 0.9), 64, 64, router=R.ROUTER_ENTROPY, kappa=0.5)
    for i in range(rt["tiers"].shape[0]):
        for j in R.diag_blocks(i, 64, 64, N):
            assert rt["tiers"][i, j] == R.TIER_FULL
        kept = (rt["tiers"][i] != R.TIER_SKIP).sum()
        assert kept >= rt["keep"][i]            # the diagonal may add one
        assert kept <= rt["keep"][i] + 1
