"""GPU parity of 32-key blocks ("FG-Attn", searcharxiv author page, abstract:
skipping at M x N sub-tiles with M >= 16 queries and N >= 1 keys; here M = 128
and N = 32).  The router works on 32-key blocks; the attention kernel packs the
kept blocks of one tier four at a time, in list order, into 128-key tiles, and
the oracle runs the same grouping (``key_pack`` = 4).  Plan parity as for the
other shapes; forward within rel-L2 1e-2 and max-abs 2e-2 of the oracle.
Ragged cases put the sequence's 22-key last block anywhere in a pack."""

import numpy as np
import pytest
import torch

from gpu_helpers import assert_out_close, compare_tiers, inputs, oracle_head, run_gpu, to64
from oracle import quant as Qz
from test_gpu_parity import _plan_parity

pytestmark = pytest.mark.gpu

CASES = [
    # N = 630: 20 key blocks, the last of 22 keys; NVFP4 low tier
    ("nvfp4 ragged", {"grid": (3, 10, 21), "H": 2}, (0, 1, 3)),
    # NVFP4 + residual on the middle-mass band (four tiers)
    ("nvfp4+res ragged", {"grid": (3, 10, 21), "H": 2, "low": Qz.LOW_NVFP4_RES,
                          "tau": (0.5, 0.675, 0.85)}, (0, 1, 2, 3)),
    # full and skipped blocks only
    ("no low tier", {"grid": (3, 10, 21), "H": 2, "low": Qz.LOW_NONE, "tau": (0.7,)}, (0, 3)),
    # N = 1536 = 48 blocks of 32, no ragged block; longer rows
    ("nvfp4 whole blocks", {"grid": (4, 16, 24), "H": 1}, (0, 1, 3)),
]


@pytest.mark.parametrize("what,over,need", CASES, ids=[c[0] for c in CASES])
def test_key_blocks_of_32_plan_and_forward(cuda_ok, what, over, need):
    cfg, Q, K, V = inputs("480p-fg", **over)
    assert cfg.block_k == 32 and cfg.key_pack == 4
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])
    t = views["tier_map"].numpy()
    for code in need:
        assert (t == code).any(), f"{what}: no tile of tier {code}"
    counts = views["row_counts"].numpy()
    assert (counts[..., :3] % 4 != 0).any()      # some tiles hold fewer than four blocks
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(t[h], rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"{what} head {h}")


def test_key_blocks_of_32_all_full_matches_sdpa(cuda_ok):
    cfg, Q, K, V = inputs("480p-fg", grid=(3, 10, 21), H=2)
    _, views, O, st = run_gpu(cfg, Q, K, V, tau=(2.0, 2.0))
    assert st == 0
    assert (views["tier_map"].numpy() == 3).all()
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.cuda().float(), K.cuda().float(), V.cuda().float()).cpu()
    rel = (O.float() - ref).norm() / ref.norm()
    assert rel < 1e-2
    _, _, Oref = oracle_head(cfg, Q, K, V, 0, 1, tau=(2.0, 2.0))
    assert_out_close(to64(O[0, 1]), Oref, "all full")


def test_key_blocks_of_32_skip_only(cuda_ok):
    # thresholds 0: the four diagonal blocks of each query block stay full,
    # every other 32-key block is replaced by its means
    cfg, Q, K, V = inputs("480p-fg", grid=(3, 10, 21), H=2)
    _, views, O, st = run_gpu(cfg, Q, K, V, tau=(0.0, 0.0))
    assert st == 0
    t = views["tier_map"].numpy()
    assert ((t == 3) | (t == 0)).all()
    assert (views["row_counts"].numpy()[..., 0] <= 4).all()
    for h in range(cfg.H):
        _, _, Oref = oracle_head(cfg, Q, K, V, 0, h, tau=(0.0, 0.0))
        assert_out_close(to64(O[0, h]), Oref, f"skip-only head {h}")


@pytest.mark.parametrize("N", [1, 17, 40, 100])
def test_key_blocks_of_32_short_sequences(cuda_ok, N):
    # sequences shorter than one 128-query block: one to four 32-key blocks,
    # the last one ragged (N = 1, 17, 40, 100), every block of the row inside
    # one packed tile with the forced diagonal
    base, Q, K, V = inputs("480p-fg", grid=(3, 10, 21), H=2)
    cfg = base.with_(grid=(1, 1, N))
    Qs, Ks, Vs = (x[:, :, :N].contiguous() for x in (Q, K, V))
    _, views, O, st = run_gpu(cfg, Qs, Ks, Vs)
    assert st == 0
    _plan_parity(cfg, Qs, Ks, Vs, views, [(0, h) for h in range(cfg.H)])
    for h in range(cfg.H):
        rt, _, Oref = oracle_head(cfg, Qs, Ks, Vs, 0, h)
        n_diff, _ = compare_tiers(views["tier_map"][h].numpy(), rt)
        assert n_diff == 0
        assert_out_close(to64(O[0, h]), Oref, f"fg N={N} head {h}")


def test_key_blocks_of_32_batch_of_two(cuda_ok):
    # B = 2 with 32-key blocks: every (b, h) routed, packed and attended
    # independently, strides over b (N = 320: ten 32-key blocks)
    cfg, Q, K, V = inputs("480p-fg", grid=(2, 10, 16), H=2, B=2)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(b, h) for b in range(2) for h in range(2)])
    for b in range(2):
        for h in range(2):
            rt, qt, Oref = oracle_head(cfg, Q, K, V, b, h)
            _, rows = compare_tiers(views["tier_map"][b * cfg.H + h].numpy(), rt)
            for i in rows:
                Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
            assert_out_close(to64(O[b, h]), Oref, f"fg batch {b} head {h}")
