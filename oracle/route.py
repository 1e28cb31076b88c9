"""Router: block pooling, pooled block softmax, cumulative-mass tiers (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

"Triage" (zhuanzhiai paper page, abstract) routes every tile from block
statistics; "HierPAS" (conference listing, abstract) estimates the attention
pattern cheaply and gives progressively reduced precision to less critical
regions; "APT" (Lattice paper summary) selects and assigns precision with two
thresholds on attention probability (APDT).  The pooled-mass router restates
these at tile level:

1. Blocks.  Query block i holds rows [i*Bq, min(N, (i+1)*Bq)); key block j
   holds keys [j*Bk, min(N, (j+1)*Bk)) and has n_j keys (ragged tails keep
   their real size).
2. Pooling.  qbar_i, kbar_j, vbar_j are fp64 means of the bf16 rows; the skip
   tier uses their bf16 (round to nearest even) copies.
3. Pooled mass.  sbar_ij = qbar_i . kbar_j * scale; M_ij = n_j exp(sbar_ij -
   max_j sbar_ij) / sum_j (.)  (each block weighted by its key count, as the
   skip tier weights block j by n_j).
4. Tiers.  Sort j by (-M_ij, j); C_r is the exclusive prefix sum of the sorted
   masses; the tile at rank r takes the most precise tier t whose threshold
   tau_t satisfies C_r < tau_t, else it is skipped (the tile that crosses a
   threshold is kept: the smallest set covering tau).  Then every key block
   whose token range meets query block i's range is made full.
5. Flags.  A tile is flagged when |C_r - tau_t| <= 1e-5 tau_t for some t, or
   when it and a sort neighbour have |M - M'| <= 1e-5 max(M, M') and got
   different tiers from the prefix rule: only there may a GPU router differ.
6. Lists.  Per row: full blocks, then residual, then low, then skip; within a
   tier in the sort order of step 4, so a row meets its heaviest blocks (and,
   nearly always, its largest logits) first.

The price router (router = ROUTER_PRICE) replaces step 4 with Triage's rule as
the abstract states it: predict each tile's error under each tier from block
statistics and move a tile to a more accurate tier only when the predicted
error reduction is worth the extra compute at a single price.  Reading:

4'. Predicted error of tile (i, j) under tier t: e_t = M_ij * eps_t, with eps
    the unit roundoff of the tier's arithmetic (bf16 2^-8; FP8 e4m3 2^-4;
    NVFP4 e2m1 2^-2; NVFP4 plus its residual 2^-4, the square of e2m1's) and,
    for skip, eps_skip = delta_ij = scale * sqrt(sum_c (qbar_ic^2 + qvar_ic)
    kvar_jc), where kvar_jc (qvar_ic) is the variance of coordinate c over key
    block j's keys (query block i's queries), the mean of (x_c - xbar_c)^2:
    the RMS over the tile's (query, key) pairs of how far a query's logit
    moves from the one it has with the block's mean key, were the
    coordinates uncorrelated; that is what replacing the block by its means
    ignores (0 when the block's keys are equal, and then skipping is exact).
    Cost of tier t: the compute the tier spends, a parameter (tier_cost, by
    tier code).  By default each tier's measured per-tile time on the fused
    kernel relative to a bf16 tile (skip 0.008, FP8 1.0, NVFP4 1.1, NVFP4 +
    residual 2.2, bf16 1.0): the abstract moves a tile up only when the
    error reduction justifies the extra compute, and the compute a tier
    costs is what the kernel spends on it.  The tile takes the tier of least
    e_t + price * cost_t among the tiers the low format provides; on a tie the
    cheaper tier.  The forced diagonal (step 4's last sentence) still applies,
    and step 6 orders the lists as before.
5'. A tile is flagged when another tier's objective is within 1e-6 (relative)
    of the chosen one's.

The entropy router (router = ROUTER_ENTROPY) follows "HierPAS" (conference
listing, abstract): retention ratios adapted across heads and blocks from an
entropy analysis of a cheap estimate of the attention pattern, and precision
reduced progressively on the less critical part.  Reading, per query block i
(its pooled distribution M_i. is the pattern estimate of step 3):

4''. H_i = -sum_j M_ij ln M_ij; the row keeps k_i = min(nKb, max(1,
     ceil(kappa exp(H_i)))) key blocks, exp(H_i) being the effective number of
     blocks it attends and kappa the retention scale.  In the (-M, j) order of
     step 4, ranks r < k_i are kept, with the precision of step 4's prefix
     rule (the most precise t with C_r < tau_t), or the least precise kept tier
     when no threshold is met; ranks r >= k_i are skipped.  The forced
     diagonal still applies.
5''. A row's tiles are flagged when kappa exp(H_i) is within 1e-9 (relative)
     of an integer, besides step 5's flags.

Plan reuse ("APT" TAFA, Lattice paper summary: attention probabilities are
predicted across diffusion timesteps from their similarity): a plan made on
the inputs of one timestep serves the next ones.  Reading: a reused step keeps
the plan's tier map, flags and lists (steps 4-6) and takes everything else
from its own inputs: the block means (so the skip tier uses the current
kbar_j, vbar_j) and the low-precision copies.
"""

from __future__ import annotations

import math

import numpy as np

from .formats import bf16_rne
from .quant import LOW_FP8, LOW_NONE, LOW_NVFP4, LOW_NVFP4_RES

TIER_SKIP, TIER_LOW, TIER_RES, TIER_FULL = 0, 1, 2, 3
FLAG_REL = 1e-5
ROUTER_MASS, ROUTER_PRICE, ROUTER_ENTROPY = 0, 1, 2
FLAG_REL_ENTROPY = 1e-9
FLAG_REL_PRICE = 1e-6


def block_ranges(N: int, block: int):
    return [(b * block, min(N, (b + 1) * block)) for b in range(-(-N // block))]


def pool_means(X: np.ndarray, block: int):
    """fp64 means of each block of rows, and the row counts n_j."""
    rngs = block_ranges(X.shape[0], block)
    means = np.stack([X[a:b].mean(axis=0) for a, b in rngs])
    counts = np.array([b - a for a, b in rngs], dtype=np.int64)
    return means, counts


def pooled_mass(qbar: np.ndarray, kbar: np.ndarray, n_k: np.ndarray, scale: float):
    """M [nQb, nKb]: n_j-weighted softmax over key blocks of pooled logits."""
    s = (qbar @ kbar.T) * scale
    w = n_k[None, :] * np.exp(s - s.max(axis=1, keepdims=True))
    return w / w.sum(axis=1, keepdims=True)


def diag_blocks(i: int, block_q: int, block_k: int, N: int):
    """Key blocks whose token range intersects query block i's token range."""
    a, b = i * block_q, min(N, (i + 1) * block_q)
    return list(range(a // block_k, (b - 1) // block_k + 1))


def tier_codes_for(tau) -> list:
    """Tier of each threshold, most precise first: (full, low) or (full, res, low)."""
    if len(tau) == 2:
        return [TIER_FULL, TIER_LOW]
    if len(tau) == 3:
        return [TIER_FULL, TIER_RES, TIER_LOW]
    if len(tau) == 1:
        return [TIER_FULL]
    raise ValueError("1 to 3 thresholds")


def assign_tiers(M_row: np.ndarray, tau, diag=()):
    """Tiers (uint8 [nKb]) and flags (bool [nKb]) of one query-block row."""
    n = M_row.shape[0]
    j = np.arange(n)
    order = np.lexsort((j, -M_row))                  # primary -M, secondary j
    Ms = M_row[order]
    C = np.concatenate([[0.0], np.cumsum(Ms)[:-1]])  # exclusive prefix
    codes = tier_codes_for(tau)
    tier_sorted = np.full(n, TIER_SKIP, dtype=np.uint8)
    for t in reversed(range(len(tau))):              # most precise tier wins
        tier_sorted[C < tau[t]] = codes[t]
    flag_sorted = np.zeros(n, dtype=bool)
    for t in range(len(tau)):
        flag_sorted |= np.abs(C - tau[t]) <= FLAG_REL * tau[t]
    if n > 1:
        near = np.abs(Ms[1:] - Ms[:-1]) <= FLAG_REL * np.maximum(Ms[1:], Ms[:-1])
        diff = tier_sorted[1:] != tier_sorted[:-1]
        pair = near & diff
        flag_sorted[1:] |= pair
        flag_sorted[:-1] |= pair
    tiers = np.empty(n, dtype=np.uint8)
    flags = np.empty(n, dtype=bool)
    tiers[order] = tier_sorted
    flags[order] = flag_sorted
    for jj in diag:
        tiers[jj] = TIER_FULL
    return tiers, flags


def assign_tiers_entropy(M_row: np.ndarray, tau, kappa: float, diag=()):
    """Tiers (uint8 [nKb]), flags (bool [nKb]) and k_i of one row by the
    entropy retention rule (step 4'')."""
    n = M_row.shape[0]
    pos = M_row[M_row > 0]
    H = float(-(pos * np.log(pos)).sum())
    want = kappa * math.exp(H)
    k = min(n, max(1, math.ceil(want)))
    tiers, flags = assign_tiers(M_row, tau)          # precision by the prefix rule
    order = np.lexsort((np.arange(n), -M_row))
    kept_low = tier_codes_for(tau)[-1]
    for r, j in enumerate(order):
        if r >= k:
            tiers[j] = TIER_SKIP
        elif tiers[j] == TIER_SKIP:
            tiers[j] = kept_low
    near = abs(want - round(want)) <= FLAG_REL_ENTROPY * max(1.0, want)
    if near:
        flags[:] = True
    for jj in diag:
        tiers[jj] = TIER_FULL
    return tiers, flags, k


def block_spread(X: np.ndarray, block: int) -> np.ndarray:
    """var [nb, d]: per block, the variance of each coordinate over its rows,
    the mean of (x_c - xbar_c)^2 (fp64, two passes)."""
    out = []
    for a, b in block_ranges(X.shape[0], block):
        dev = X[a:b] - X[a:b].mean(axis=0)
        out.append((dev * dev).mean(axis=0))
    return np.stack(out)


def default_tier_cost(low: int):
    """Step 4' costs when none are given, by tier code (skip, low, res, full):
    each tier's per-tile time on the fused attention kernel, relative to a
    bf16 tile (a skipped block: one column of a 128-block skip chunk)."""
    return (0.008, 1.0 if low == LOW_FP8 else 1.1, 2.2, 1.0)


def price_tiers(low: int, tier_cost=None):
    """(tier, eps, cost) of the tiers the low format provides, cheapest first;
    eps None marks skip, whose error factor is the tile's delta (step 4').
    ``tier_cost`` by tier code (skip, low, res, full); None or all zero: the
    defaults."""
    if tier_cost is None or not any(tier_cost):
        tier_cost = default_tier_cost(low)
    c = [float(x) for x in tier_cost]
    skip, full = (TIER_SKIP, None, c[TIER_SKIP]), (TIER_FULL, 2.0 ** -8, c[TIER_FULL])
    if low == LOW_NONE:
        return [skip, full]
    if low == LOW_FP8:
        return [skip, (TIER_LOW, 2.0 ** -4, c[TIER_LOW]), full]
    if low == LOW_NVFP4:
        return [skip, (TIER_LOW, 2.0 ** -2, c[TIER_LOW]), full]
    if low == LOW_NVFP4_RES:
        return [skip, (TIER_LOW, 2.0 ** -2, c[TIER_LOW]), (TIER_RES, 2.0 ** -4, c[TIER_RES]), full]
    raise ValueError("unknown low format")


def assign_tiers_price(M_row: np.ndarray, delta_row: np.ndarray, price: float, low: int,
                       diag=(), tier_cost=None):
    """Tiers (uint8 [nKb]) and flags (bool [nKb]) of one row by the price rule."""
    n = M_row.shape[0]
    table = price_tiers(low, tier_cost)
    tiers = np.empty(n, dtype=np.uint8)
    flags = np.zeros(n, dtype=bool)
    for j in range(n):
        objs = [M_row[j] * (delta_row[j] if eps is None else eps) + price * cost
                for _, eps, cost in table]
        best = 0
        for t in range(1, len(objs)):
            if objs[t] < objs[best]:
                best = t
        tiers[j] = table[best][0]
        for t in range(len(objs)):
            if t != best and abs(objs[t] - objs[best]) <= FLAG_REL_PRICE * max(abs(objs[t]), abs(objs[best])):
                flags[j] = True
    for jj in diag:
        tiers[jj] = TIER_FULL
    return tiers, flags


def row_lists(tiers_row: np.ndarray, M_row: np.ndarray):
    """counts [full, res, low, skip] and the key-block list in that tier order;
    within a tier, blocks follow the router's (-M, j) order (largest pooled
    mass first, lower j first among equal masses)."""
    order = np.lexsort((np.arange(len(M_row)), -M_row))
    groups = [order[tiers_row[order] == t] for t in (TIER_FULL, TIER_RES, TIER_LOW, TIER_SKIP)]
    counts = np.array([len(g) for g in groups], dtype=np.int32)
    return counts, np.concatenate(groups).astype(np.int32)


def route_head(Qh, Kh, Vh, tau, block_q: int, block_k: int, scale: float = 0.0,
               keep_diag_full: bool = True, router: int = ROUTER_MASS, price: float = 0.0,
               low: int = LOW_NVFP4, kappa: float = 1.0, tier_cost=None) -> dict:
    """Router output for one head (fp64 values of bf16 Q, K, V [N, d]).
    ``router`` ROUTER_MASS uses ``tau`` (steps 4-5); ROUTER_PRICE uses
    ``price`` and the tiers of ``low`` (steps 4'-5'); ROUTER_ENTROPY uses
    ``kappa`` and ``tau`` (steps 4''-5'')."""
    N, d = Qh.shape
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    qbar, _ = pool_means(Qh, block_q)
    kbar, n_k = pool_means(Kh, block_k)
    vbar, _ = pool_means(Vh, block_k)
    M = pooled_mass(qbar, kbar, n_k, scale)
    kvar = block_spread(Kh, block_k)
    qvar = block_spread(Qh, block_q)
    delta = scale * np.sqrt((qbar * qbar + qvar) @ kvar.T)
    nqb, nkb = M.shape
    tiers = np.empty((nqb, nkb), dtype=np.uint8)
    flags = np.empty((nqb, nkb), dtype=bool)
    counts = np.empty((nqb, 4), dtype=np.int32)
    lists = np.empty((nqb, nkb), dtype=np.int32)
    keep = np.full(nqb, nkb, dtype=np.int64)
    for i in range(nqb):
        diag = diag_blocks(i, block_q, block_k, N) if keep_diag_full else ()
        if router == ROUTER_PRICE:
            tiers[i], flags[i] = assign_tiers_price(M[i], delta[i], price, low, diag, tier_cost)
        elif router == ROUTER_ENTROPY:
            tiers[i], flags[i], keep[i] = assign_tiers_entropy(M[i], tau, kappa, diag)
        else:
            tiers[i], flags[i] = assign_tiers(M[i], tau, diag)
        counts[i], lists[i] = row_lists(tiers[i], M[i])
    return {"qbar": qbar, "kbar": kbar, "vbar": vbar, "n_k": n_k, "M": M,
            "kvar": kvar, "qvar": qvar, "delta": delta, "keep": keep,
            "kbar_b": bf16_rne(kbar), "vbar_b": bf16_rne(vbar), "scale": scale,
            "tiers": tiers, "flags": flags, "counts": counts, "lists": lists}


def reuse_plan(rt_plan: dict, Qh, Kh, Vh, block_q: int, block_k: int, scale: float = 0.0) -> dict:
    """Router output for the current inputs under a plan made on earlier ones:
    ``rt_plan``'s tiers, flags, counts and lists; the current block means."""
    N, d = Qh.shape
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    qbar, _ = pool_means(Qh, block_q)
    kbar, n_k = pool_means(Kh, block_k)
    vbar, _ = pool_means(Vh, block_k)
    out = dict(rt_plan)
    out.update({"qbar": qbar, "kbar": kbar, "vbar": vbar, "n_k": n_k,
                "M": pooled_mass(qbar, kbar, n_k, scale),
                "kbar_b": bf16_rne(kbar), "vbar_b": bf16_rne(vbar), "scale": scale})
    return out
