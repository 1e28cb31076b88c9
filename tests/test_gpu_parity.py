"""GPU parity: the CUDA path through the C ABI against the oracle.

Plan stage: block means (fp64) and their bf16 copies bit-exact; FP8 / NVFP4
(+residual) codes, scales and dequantised values bit-exact; pooled logits and
masses to fp64 rounding; the tier map bit-exact except on oracle-flagged tiles;
the row lists consistent with the tier map.  Forward: O within rel-L2 1e-2 and
max-abs 2e-2 of the oracle run on the same inputs with the same rounding rules
(rows whose tier map matches the oracle's).
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (assert_out_close, check_lists, check_vt, compare_tiers, inputs,
                         oracle_head, run_gpu, to64, unpack_fp4)
from oracle import quant as Qz

pytestmark = pytest.mark.gpu


def _plan_parity(cfg, Q, K, V, views, heads):
    nkb = cfg.n_kb
    n_k = views["n_k"].numpy()
    np.testing.assert_array_equal(n_k, [min(cfg.block_k, cfg.N - j * cfg.block_k) for j in range(nkb)])
    for (b, h) in heads:
        bh = b * cfg.H + h
        rt, qt, _ = oracle_head(cfg, Q, K, V, b, h, qblocks=[])
        np.testing.assert_array_equal(views["qbar"][bh].numpy(), rt["qbar"])
        np.testing.assert_array_equal(views["kbar"][bh].numpy(), rt["kbar"])
        np.testing.assert_array_equal(to64(views["kbar_b"][bh]), rt["kbar_b"])
        np.testing.assert_array_equal(to64(views["vbar_b"][bh]), rt["vbar_b"])
        np.testing.assert_allclose(views["logits"][bh].numpy(), (rt["qbar"] @ rt["kbar"].T) * rt["scale"],
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(views["mass"][bh].numpy(), rt["M"], rtol=1e-10, atol=1e-15)
        if getattr(cfg, "router", 0) == 1:
            # the price router's block statistics: key-block coordinate
            # variances and the skip tier's predicted error factor
            np.testing.assert_allclose(views["kvar"][bh].numpy(), rt["kvar"], rtol=1e-12, atol=0)
            np.testing.assert_allclose(views["qvar"][bh].numpy(), rt["qvar"], rtol=1e-12, atol=0)
            np.testing.assert_allclose(views["spread"][bh].numpy(), rt["delta"], rtol=1e-12, atol=0)
        tiers = views["tier_map"][bh].numpy()
        compare_tiers(tiers, rt)
        check_lists(tiers, views["row_counts"][bh].numpy(), views["row_lists"][bh].numpy(),
                    views["mass"][bh].numpy())
        # and equal to the oracle's lists wherever the tier rows agree
        same = (tiers == rt["tiers"]).all(axis=1)
        np.testing.assert_array_equal(views["row_lists"][bh].numpy()[same], rt["lists"][same])
        if cfg.low == Qz.LOW_FP8:
            for t in "qkv":
                np.testing.assert_array_equal(views[f"{t}_codes"][bh].numpy(), qt[f"{t}_codes"])
                np.testing.assert_array_equal(views[f"{t}_scales"][bh].numpy().astype(np.float64), qt[f"{t}_scale"])
                if f"d{t}" in views:   # no bf16 images are kept (the views are absent)
                    np.testing.assert_array_equal(to64(views[f"d{t}"][bh]), qt[f"d{t}"][:cfg.N])
        elif cfg.low in (Qz.LOW_NVFP4, Qz.LOW_NVFP4_RES):
            pres = ["", "r"] if cfg.low == Qz.LOW_NVFP4_RES else [""]
            for pre in pres:
                for t in "qk":
                    np.testing.assert_array_equal(unpack_fp4(views[f"{pre}{t}_codes"][bh].numpy()),
                                                  qt[f"{pre}{t}_codes"])
                    np.testing.assert_array_equal(views[f"{pre}{t}_scales"][bh].numpy(), qt[f"{pre}{t}_sc"])
                check_vt(views[f"{pre}v_codes"][bh].numpy(), views[f"{pre}v_scales"][bh].numpy(),
                         qt[f"{pre}v_codes"], qt[f"{pre}v_sc"])
            for t in "qkv":
                if f"d{t}" in views:   # no bf16 images are kept (the views are absent)
                    np.testing.assert_array_equal(to64(views[f"d{t}"][bh]), qt[f"d{t}"][:cfg.N])
            if cfg.low == Qz.LOW_NVFP4_RES:
                for t, key in (("q", "rq"), ("k", "rk"), ("v", "rv")):
                    if f"dr{t}" in views:
                        np.testing.assert_array_equal(to64(views[f"dr{t}"][bh]), qt[key][:cfg.N])


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_plan_parity_fp8(cuda_ok, name):
    cfg, Q, K, V = inputs(name)
    _, views, _, st = run_gpu(cfg, Q, K, V, forward=False)
    assert st == 0
    heads = [(0, h) for h in range(cfg.H)]
    _plan_parity(cfg, Q, K, V, views, heads)


def test_plan_parity_nvfp4_ragged(cuda_ok):
    # 480p tile / format settings on a smaller ragged grid (N = 3*10*21 = 630 = 4*128 + 118)
    cfg, Q, K, V = inputs("480p", grid=(3, 10, 21), H=3)
    _, views, _, st = run_gpu(cfg, Q, K, V, forward=False)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])


def test_plan_parity_nvfp4_residual_ragged(cuda_ok):
    cfg, Q, K, V = inputs("720p", grid=(3, 9, 20), H=2)   # N = 540 = 4*128 + 28
    _, views, _, st = run_gpu(cfg, Q, K, V, forward=False)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_forward_parity_fp8(cuda_ok, name):
    cfg, Q, K, V = inputs(name)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    heads = [(0, h) for h in range(cfg.H)] if cfg.H <= 2 else [(0, 0), (0, cfg.H // 2), (0, cfg.H - 1)]
    for (b, h) in heads:
        bh = b * cfg.H + h
        rt, qt, Oref = oracle_head(cfg, Q, K, V, b, h)
        _, rows = compare_tiers(views["tier_map"][bh].numpy(), rt)
        Og = to64(O[b, h])
        for i in rows:  # a flagged tile differs: compare only rows routed alike
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(Og, Oref, f"{name} head {h}")


def test_forward_parity_nvfp4_ragged(cuda_ok):
    cfg, Q, K, V = inputs("480p", grid=(3, 10, 21), H=3)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"nvfp4 head {h}")


def test_plan_and_forward_parity_fp8_native_ragged(cuda_ok):
    # sweep settings (FP8 e4m3 low tier on 128 x 128 tiles, d = 128: the FP8
    # tensor-pipe path) on a ragged grid, N = 3*10*21 = 630
    cfg, Q, K, V = inputs("sweep70", grid=(3, 10, 21), H=3)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])
    t = views["tier_map"].numpy()
    assert (t == 1).any() and (t == 3).any()
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"fp8 native head {h}")


def test_forward_parity_nvfp4_residual_ragged(cuda_ok):
    # four tiers: full, NVFP4 + residual, NVFP4, skip (720p settings, N = 540)
    cfg, Q, K, V = inputs("720p", grid=(3, 9, 20), H=2)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    t = views["tier_map"].numpy()
    assert (t == 2).any() and (t == 1).any() and (t == 0).any()
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"nvfp4+res head {h}")


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_all_full_matches_oracle_and_sdpa(cuda_ok, name):
    cfg, Q, K, V = inputs(name)
    _, views, O, st = run_gpu(cfg, Q, K, V, tau=(2.0, 2.0))
    assert st == 0
    assert (views["tier_map"].numpy() == 3).all()
    for h in range(min(cfg.H, 2)):
        _, _, Oref = oracle_head(cfg, Q, K, V, 0, h, tau=(2.0, 2.0))
        assert_out_close(to64(O[0, h]), Oref, f"all-full head {h}")
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.cuda().float(), K.cuda().float(), V.cuda().float()).cpu()
    rel = (O.float() - ref).norm() / ref.norm()
    assert rel < 1e-2


def test_skip_only_rows(cuda_ok):
    # thresholds 0: only the diagonal stays (full), every other tile is a skip
    cfg, Q, K, V = inputs("tiny")
    _, views, O, st = run_gpu(cfg, Q, K, V, tau=(0.0, 0.0))
    assert st == 0
    t = views["tier_map"].numpy()
    assert ((t == 3) | (t == 0)).all() and (t == 0).any()
    for h in range(cfg.H):
        rt, _, Oref = oracle_head(cfg, Q, K, V, 0, h, tau=(0.0, 0.0))
        assert_out_close(to64(O[0, h]), Oref, f"skip-only head {h}")


def _forward_parity(cfg, Q, K, V, what, need_tiers=()):
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])
    t = views["tier_map"].numpy()
    for code in need_tiers:
        assert (t == code).any(), f"{what}: no tile of tier {code}"
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"{what} head {h}")


def test_forward_parity_d128_query_blocks_of_64(cuda_ok):
    # d = 128 with 64-row query blocks and 128-key tiles: native FP8 tiles in
    # the 16-warp kernel, whose TMEM lanes of rows 64..127 carry no query rows
    cfg, Q, K, V = inputs("sweep70", grid=(3, 10, 21), H=2, block_q=64)
    _forward_parity(cfg, Q, K, V, "d128 bq64", need_tiers=(1, 3))


def test_forward_parity_d128_key_blocks_of_64(cuda_ok):
    # d = 128 with 128-row query blocks and 64-key tiles (two column parts of S)
    cfg, Q, K, V = inputs("sweep70", grid=(3, 10, 21), H=2, block_k=64)
    _forward_parity(cfg, Q, K, V, "d128 bk64", need_tiers=(1, 3))


def test_forward_parity_no_low_tier(cuda_ok):
    # one threshold: full and skipped tiles only (d = 128, 128 x 128 tiles)
    cfg, Q, K, V = inputs("sweep70", grid=(3, 10, 21), H=2, low=0, tau=(0.7,))
    _forward_parity(cfg, Q, K, V, "no low tier", need_tiers=(0, 3))


def test_all_full_d128_matches_sdpa(cuda_ok):
    # every tile full at d = 128: the bf16 path against torch's own attention
    cfg, Q, K, V = inputs("480p", grid=(3, 10, 21), H=3)
    _, views, O, st = run_gpu(cfg, Q, K, V, tau=(2.0, 2.0))
    assert st == 0
    assert (views["tier_map"].numpy() == 3).all()
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.cuda().float(), K.cuda().float(), V.cuda().float()).cpu()
    rel = (O.float() - ref).norm() / ref.norm()
    assert rel < 1e-2


# nominal tensor-pipe rates (by tier code: skip, low, res, full): every tier
# of the low format has a use, so the test meets all of them
NOMINAL_NVFP4 = (0.0, 1.0, 3.0, 4.0)
NOMINAL_FP8 = (0.0, 2.0, 3.0, 4.0)


@pytest.mark.parametrize("name,grid,price,cost,n_tiers", [
    ("480p-price", (3, 10, 21), 0.028, NOMINAL_NVFP4, 3),  # bf16, NVFP4 + residual, NVFP4, skip
    ("480p", (3, 10, 21), 0.04, NOMINAL_NVFP4, 3),         # NVFP4 low tier
    ("sweep70", (3, 10, 21), 0.06, NOMINAL_FP8, 3),        # native FP8 low tier
    ("small", None, 0.002, NOMINAL_FP8, 3),                # FP8 low tier, d = 64, 64-key tiles
    ("480p-price", (3, 10, 21), 0.05, (0.0, 0.0, 0.0, 0.0), 2),   # the default (measured) costs
])
def test_price_router_parity(cuda_ok, name, grid, price, cost, n_tiers):
    over = {"H": 3, "router": 1, "price": price, "tier_cost": cost}
    if grid is not None:
        over["grid"] = grid
    cfg, Q, K, V = inputs(name, **over)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    t = views["tier_map"].numpy()
    assert len(np.unique(t)) >= n_tiers
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"price router {name} head {h}")


def test_plan_reuse_parity(cuda_ok):
    # a plan made on timestep 0 serves timestep 2 of a slowly changing
    # sequence: tiers and lists from step 0, block means and low copies from step 2
    import precision_attention_video_b200 as pav
    from latent_gen import get_config
    from latent_gen.generator import make_qkv_steps
    from oracle import route as Rt
    from oracle.attention import tiered_attention_head
    cfg = get_config("480p").with_(H=2, grid=(3, 10, 21))
    seq = make_qkv_steps(cfg, 3, rho=0.95)
    dev = torch.device("cuda:0")
    p = pav.params_for(cfg)
    ws = pav.alloc_workspace(p, dev)
    Q0, K0, V0 = (x.to(dev) for x in seq[0])
    pav.plan(p, Q0, K0, V0, ws)
    Q2, K2, V2 = (x.to(dev) for x in seq[2])
    pav.prep(p, Q2, K2, V2, ws)
    O = torch.empty_like(Q2)
    pav.forward(p, Q2, K2, V2, ws, O)
    torch.cuda.synchronize()
    assert pav.get_status(ws) == 0
    views = {k: v.cpu() for k, v in pav.plan_views(p, ws).items()}
    for h in range(cfg.H):
        s0 = [to64(x[0, h]) for x in seq[0]]
        s2 = [to64(x[0, h]) for x in seq[2]]
        rt0 = Rt.route_head(*s0, cfg.tau, cfg.block_q, cfg.block_k)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt0)
        ru = Rt.reuse_plan(rt0, *s2, cfg.block_q, cfg.block_k)
        np.testing.assert_array_equal(to64(views["kbar_b"][h]), ru["kbar_b"])
        np.testing.assert_array_equal(to64(views["vbar_b"][h]), ru["vbar_b"])
        qt = Qz.quantize_head(*s2, cfg.low, cfg.block_q, cfg.block_k)
        for t in "qk":
            np.testing.assert_array_equal(unpack_fp4(views[f"{t}_codes"][h].numpy()), qt[f"{t}_codes"])
        check_vt(views["v_codes"][h].numpy(), views["v_scales"][h].numpy(), qt["v_codes"], qt["v_sc"])
        Oref = tiered_attention_head(*s2, ru, qt, cfg.low, cfg.block_q, cfg.block_k,
                                     cfg.p_offset_log2, ru["scale"], False)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"plan reuse head {h}")


@pytest.mark.parametrize("name,grid,kappa", [
    ("480p", (3, 10, 21), 0.5),          # NVFP4 low tier
    ("720p", (3, 9, 20), 1.0),           # four tiers
    ("sweep70", (3, 10, 21), 0.5),       # native FP8 low tier
    ("small", None, 0.5),                # FP8 low tier, d = 64, 64-key tiles
])
def test_entropy_router_parity(cuda_ok, name, grid, kappa):
    over = {"H": 2, "router": 2, "kappa": kappa}
    if grid is not None:
        over["grid"] = grid
    cfg, Q, K, V = inputs(name, **over)
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    t = views["tier_map"].numpy()
    assert len(np.unique(t)) >= 3
    _plan_parity(cfg, Q, K, V, views, [(0, h) for h in range(cfg.H)])
    for h in range(cfg.H):
        rt, qt, Oref = oracle_head(cfg, Q, K, V, 0, h)
        _, rows = compare_tiers(views["tier_map"][h].numpy(), rt)
        for i in rows:
            Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
        assert_out_close(to64(O[0, h]), Oref, f"entropy router {name} head {h}")


def test_forward_parity_batch_of_two(cuda_ok):
    # B = 2: every (b, h) routed and attended independently, strides over b
    cfg, Q, K, V = inputs("480p", grid=(2, 10, 16), H=2, B=2)   # N = 320 = 2*128 + 64
    _, views, O, st = run_gpu(cfg, Q, K, V)
    assert st == 0
    _plan_parity(cfg, Q, K, V, views, [(b, h) for b in range(2) for h in range(2)])
    for b in range(2):
        for h in range(2):
            rt, qt, Oref = oracle_head(cfg, Q, K, V, b, h)
            _, rows = compare_tiers(views["tier_map"][b * cfg.H + h].numpy(), rt)
            for i in rows:
                Oref[i * cfg.block_q:(i + 1) * cfg.block_q] = np.nan
            assert_out_close(to64(O[b, h]), Oref, f"batch {b} head {h}")


def test_head_interleaved_layout_matches_contiguous(cuda_ok):
    # Q, K, V, O stored [B, N, H, d] (heads interleaved per token) and passed
    # with their strides: the same plan and output, bit for bit, as the
    # contiguous [B, H, N, d] run
    import precision_attention_video_b200 as pav
    cfg, Q, K, V = inputs("480p", grid=(3, 10, 21), H=3)
    _, views1, O1, st1 = run_gpu(cfg, Q, K, V)
    assert st1 == 0
    dev = torch.device("cuda:0")
    Qs, Ks, Vs = (x.permute(0, 2, 1, 3).contiguous().to(dev).permute(0, 2, 1, 3) for x in (Q, K, V))
    assert Qs.stride() == (cfg.N * cfg.H * cfg.d, cfg.d, cfg.H * cfg.d, 1)
    p = pav.params_for(cfg, strides=Qs.stride()[:3])
    ws = pav.alloc_workspace(p, dev)
    pav.plan(p, Qs, Ks, Vs, ws)
    Os = torch.empty_like(Qs)
    assert Os.stride() == Qs.stride()
    pav.forward(p, Qs, Ks, Vs, ws, Os)
    torch.cuda.synchronize()
    assert pav.get_status(ws) == 0
    views = {k: v.cpu() for k, v in pav.plan_views(p, ws).items()}
    for k in ("tier_map", "row_counts", "row_lists", "qbar", "kbar", "q_codes", "k_codes", "v_codes",
              "q_scales", "k_scales", "v_scales"):
        assert torch.equal(views[k], views1[k]), k
    assert torch.equal(Os.cpu(), O1)


@pytest.mark.parametrize("name,N", [("tiny", 1), ("tiny", 17), ("tiny", 100), ("480p", 1),
                                    ("480p", 17), ("480p", 100), ("720p", 40)])
def test_sequences_shorter_than_one_tile(cuda_ok, name, N):
    # sequences shorter than one 128-token tile: N = 1 (a single key, and one
    # NVFP4 V group holding one token), N = 17 (one group and one token of the
    # next), N = 100 and 40 (a block short of its 128 rows; with 64-token
    # blocks, N = 100 is a full block and a 36-token tail); the inputs are the
    # first N tokens of the seeded ragged-grid inputs
    grid = {"tiny": (4, 16, 16), "480p": (3, 10, 21), "720p": (3, 9, 20)}[name]
    base, Q, K, V = inputs(name, grid=grid, H=2)
    cfg = base.with_(grid=(1, 1, N))
    Qs, Ks, Vs = (x[:, :, :N].contiguous() for x in (Q, K, V))
    _, views, O, st = run_gpu(cfg, Qs, Ks, Vs)
    assert st == 0
    _plan_parity(cfg, Qs, Ks, Vs, views, [(0, h) for h in range(cfg.H)])
    for h in range(cfg.H):
        rt, _, Oref = oracle_head(cfg, Qs, Ks, Vs, 0, h)
        n_diff, _ = compare_tiers(views["tier_map"][h].numpy(), rt)
        assert n_diff == 0
        assert_out_close(to64(O[0, h]), Oref, f"{name} N={N} head {h}")


@pytest.mark.parametrize("name,over", [
    # rows of 512 key blocks (480p with 64-key blocks): the one-CTA-a-row router
    ("480p", {"H": 1, "block_k": 64}),
    ("480p", {"H": 1, "block_k": 64, "router": 1, "price": 0.004, "tier_cost": (0.0, 1.0, 3.0, 4.0)}),
    ("480p", {"H": 1, "block_k": 64, "router": 2, "kappa": 0.7}),
    # rows of 929 key blocks (720p, four tiers)
    ("720p", {"H": 1}),
    ("720p", {"H": 1, "router": 2, "kappa": 1.0}),
])
def test_long_row_router_parity(cuda_ok, name, over):
    # the router for rows of more than 256 key blocks (one CTA a row): tier
    # maps, counts and lists against the oracle, on whole heads
    cfg, Q, K, V = inputs(name, **over)
    _, views, _, st = run_gpu(cfg, Q, K, V, forward=False)
    assert st == 0
    assert len(np.unique(views["tier_map"].numpy())) >= 2
    _plan_parity(cfg, Q, K, V, views, [(0, 0)])


def test_long_row_router_orders_masses_that_share_a_float(cuda_ok):
    # The router of rows longer than 256 key blocks sorts on the float of
    # each block's mass (then j) and repairs the order among masses that
    # round to the same float.  Here 40 key blocks differ only in one
    # coordinate of one key, which the queries weigh by 2^-12: their masses
    # differ by about 3e-9 relative (one float), and increase with j, so the
    # float sort alone would list them in the wrong order.
    nkb, d = 300, 128
    N = nkb * 128
    cfg = inputs("480p", grid=(3, 10, 21), H=1)[0].with_(grid=(1, 1, N), H=1)
    rng = np.random.default_rng(5)
    base = np.round(rng.normal(size=d) * 0.5 * 128) / 128
    base[0] = 1.0
    K = np.tile(base, (N, 1)) + np.round(rng.normal(size=(N, d)) * 0.01 * 256) / 256
    K[:, 0] = 1.0
    g0 = 100
    for u in range(40):                        # the near-tied group: blocks g0 .. g0 + 39
        blk = slice((g0 + u) * 128, (g0 + u + 1) * 128)
        K[blk] = K[g0 * 128:(g0 + 1) * 128]      # a copy of block g0 ...
        K[(g0 + u) * 128, 0] = 1.0 + u * 2.0 ** -6   # ... but for one coordinate of one key
    Qm = np.round(rng.normal(size=(N, d)) * 256) / 256
    Qm[:, 0] = 2.0 ** -12
    V = rng.normal(size=(N, d))
    to_bf16 = lambda a: torch.from_numpy(a).to(torch.bfloat16).reshape(1, 1, N, d)
    Q, Kt, Vt = to_bf16(Qm), to_bf16(K), to_bf16(V)
    _, views, _, st = run_gpu(cfg, Q, Kt, Vt, forward=False)
    assert st == 0
    # the group's masses: distinct doubles, one float at most a few
    mass = views["mass"][0].numpy()
    grp = mass[0, g0:g0 + 40]
    assert len(np.unique(grp)) > 30 and len(np.unique(grp.astype(np.float32))) <= 4
    _plan_parity(cfg, Q, Kt, Vt, views, [(0, 0)])
