"""Pins of the oracle's router: pooled mass, tier sets, flags, lists."""

import itertools
import math

import numpy as np
import pytest

from oracle import route as R


def test_pool_means_ragged():
    rng = np.random.default_rng(0)
    X = rng.normal(size=(200, 16))
    m, n = R.pool_means(X, 64)
    np.testing.assert_array_equal(n, [64, 64, 64, 8])
    np.testing.assert_allclose(m[3], X[192:].sum(0) / 8, rtol=0, atol=1e-15)


def test_mass_sums_to_one_and_uniform_case():
    rng = np.random.default_rng(1)
    qbar, kbar = rng.normal(size=(5, 8)), rng.normal(size=(7, 8))
    n = np.array([64] * 6 + [8])
    M = R.pooled_mass(qbar, kbar, n, 0.3)
    np.testing.assert_allclose(M.sum(1), 1.0, rtol=0, atol=1e-14)
    # equal pooled logits -> mass proportional to key counts: n_j / N
    M0 = R.pooled_mass(np.zeros((2, 8)), kbar, n, 0.3)
    np.testing.assert_allclose(M0, np.broadcast_to(n / n.sum(), M0.shape), rtol=0, atol=1e-15)


def test_diag_blocks():
    assert R.diag_blocks(0, 64, 64, 1024) == [0]
    assert R.diag_blocks(3, 128, 64, 8192) == [6, 7]          # Bq = 2 Bk
    assert R.diag_blocks(255, 128, 128, 32760) == [255]       # ragged tail
    assert R.diag_blocks(1, 64, 128, 200) == [0]
    assert R.diag_blocks(2, 96, 64, 250) == [3]               # rows 192..249 -> blocks 3
    assert R.diag_blocks(1, 96, 64, 250) == [1, 2]            # rows 96..191


def _min_cover(M, tau):
    """Smallest k such that some k-subset of masses sums to >= tau (brute force)."""
    n = len(M)
    for k in range(0, n + 1):
        for sub in itertools.combinations(range(n), k):
            if sum(M[list(sub)]) >= tau:
                return k
    return n


def _brute_rows(rng, n, ties):
    if ties:
        base = rng.integers(1, 4, size=n).astype(float)
    else:
        base = rng.uniform(0.01, 1.0, size=n)
    return base / base.sum()


@pytest.mark.parametrize("ties", [False, True])
def test_tier_sets_against_brute_force(ties):
    rng = np.random.default_rng(2 + ties)
    for _ in range(150):
        n = int(rng.integers(2, 10))
        M = _brute_rows(rng, n, ties)
        t_full = float(rng.uniform(0.05, 0.8))
        t_low = float(rng.uniform(t_full, 0.99))
        tiers, _ = R.assign_tiers(M, (t_full, t_low))
        full = np.nonzero(tiers == R.TIER_FULL)[0]
        kept = np.nonzero(tiers >= R.TIER_LOW)[0]
        # exclusive prefix: the tile crossing tau is kept -> smallest covering set
        k_full = _min_cover(M, t_full)
        k_low = _min_cover(M, t_low)
        # the rule never keeps fewer than one block (C_0 = 0 < tau)
        assert len(full) == max(k_full, 1)
        assert len(kept) == max(k_low, 1)
        # and it takes the largest masses, lower j first among equal masses
        order = sorted(range(n), key=lambda j: (-M[j], j))
        assert sorted(order[:len(full)]) == list(full)
        assert sorted(order[:len(kept)]) == list(kept)


def test_diag_forced_full_does_not_displace():
    M = np.array([0.5, 0.3, 0.15, 0.05])
    tiers, _ = R.assign_tiers(M, (0.6, 0.9), diag=[3])
    # prefix C = [0, .5, .8, .95] -> full, full, low, skip; diagonal 3 forced full
    np.testing.assert_array_equal(tiers, [3, 3, 1, 3])


def test_three_thresholds():
    M = np.array([0.4, 0.2, 0.15, 0.1, 0.1, 0.05])
    tiers, _ = R.assign_tiers(M, (0.5, 0.675, 0.85))
    # C = [0, .4, .6, .75, .85, .95]: full, full, res, low, skip(0.85 not < 0.85), skip
    np.testing.assert_array_equal(tiers, [3, 3, 2, 1, 0, 0])


def test_flags():
    M = np.array([0.5, 0.25, 0.25])
    tiers, flags = R.assign_tiers(M, (0.5, 0.9))
    # C = [0, 0.5, 0.75]: block 1 sits exactly on tau_full -> flagged
    assert flags[1] and not flags[0]
    # near tie across a tier boundary is flagged on both tiles
    M = np.array([0.4, 0.3, 0.3 * (1 - 3e-6)])
    M = M / M.sum()
    tiers, flags = R.assign_tiers(M, (0.6, 0.99))
    assert tiers[1] != tiers[2]
    assert flags[1] and flags[2]


def test_row_lists():
    tiers = np.array([0, 3, 1, 2, 3, 0, 1], dtype=np.uint8)
    M = np.array([0.05, 0.2, 0.1, 0.15, 0.3, 0.05, 0.15])
    counts, lst = R.row_lists(tiers, M)
    np.testing.assert_array_equal(counts, [2, 1, 2, 2])
    # full: 4 (0.3), 1 (0.2); res: 3; low: 6 (0.15), 2 (0.1); skip: 0, 5 (tie, lower j first)
    np.testing.assert_array_equal(lst, [4, 1, 3, 6, 2, 0, 5])


def test_route_head_scale_and_shapes():
    rng = np.random.default_rng(5)
    X = rng.normal(size=(300, 64))
    rt = R.route_head(X, X, X, (0.6, 0.9), 128, 64)
    assert rt["scale"] == 1.0 / math.sqrt(64)
    assert rt["tiers"].shape == (3, 5)
    for i in range(3):
        assert sorted(rt["lists"][i]) == list(range(5))
        for j in R.diag_blocks(i, 128, 64, 300):
            assert rt["tiers"][i, j] == R.TIER_FULL
