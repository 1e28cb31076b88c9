"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (whole layer: every head, every query block), checked on
sampled heads and query blocks that the oracle computes one by one: the tier
map, counts and lists of whole heads, the low-precision copies of whole heads,
and the output rows of the first, a middle and the ragged last query block.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (assert_out_close, check_lists, check_vt, compare_tiers, oracle_head,
                         router_kwargs, to64, unpack_fp4)
from latent_gen import get_config, make_qkv
from oracle import quant as Qz
from oracle import route as Rt
from oracle.attention import tiered_attention_head

pytestmark = pytest.mark.gpu


def _run_full(name):
    import precision_attention_video_b200 as pav
    cfg = get_config(name)
    Q, K, V = make_qkv(cfg)
    dev = torch.device("cuda:0")
    Qd, Kd, Vd = (x.to(dev) for x in (Q, K, V))
    p = pav.params_for(cfg)
    ws = pav.alloc_workspace(p, dev)
    O = torch.empty_like(Qd)
    pav.plan(p, Qd, Kd, Vd, ws)
    pav.forward(p, Qd, Kd, Vd, ws, O)
    torch.cuda.synchronize()
    assert pav.get_status(ws) == 0
    return cfg, Q, K, V, pav.plan_views(p, ws), O


def _check_head(cfg, Q, K, V, views, O, h, qblocks):
    Qh, Kh, Vh = to64(Q[0, h]), to64(K[0, h]), to64(V[0, h])
    rt = Rt.route_head(Qh, Kh, Vh, cfg.tau, cfg.block_q, cfg.block_k, **router_kwargs(cfg))
    if getattr(cfg, "router", 0) == Rt.ROUTER_PRICE:
        np.testing.assert_allclose(views["kvar"][h].cpu().numpy(), rt["kvar"], rtol=1e-12, atol=0)
        np.testing.assert_allclose(views["qvar"][h].cpu().numpy(), rt["qvar"], rtol=1e-12, atol=0)
        np.testing.assert_allclose(views["spread"][h].cpu().numpy(), rt["delta"], rtol=1e-12, atol=0)
    tiers = views["tier_map"][h].cpu().numpy()
    _, rows = compare_tiers(tiers, rt)
    check_lists(tiers, views["row_counts"][h].cpu().numpy(), views["row_lists"][h].cpu().numpy(),
                views["mass"][h].cpu().numpy())
    np.testing.assert_array_equal(to64(views["kbar_b"][h].cpu()), rt["kbar_b"])
    np.testing.assert_array_equal(to64(views["vbar_b"][h].cpu()), rt["vbar_b"])
    qt = Qz.quantize_head(Qh, Kh, Vh, cfg.low, cfg.block_q, cfg.block_k)
    if cfg.low == Qz.LOW_FP8:
        for t in "qkv":
            np.testing.assert_array_equal(views[f"{t}_codes"][h].cpu().numpy(), qt[f"{t}_codes"])
    else:
        pres = ["", "r"] if cfg.low == Qz.LOW_NVFP4_RES else [""]
        for pre in pres:
            for t in "qk":
                np.testing.assert_array_equal(unpack_fp4(views[f"{pre}{t}_codes"][h].cpu().numpy()),
                                              qt[f"{pre}{t}_codes"])
                np.testing.assert_array_equal(views[f"{pre}{t}_scales"][h].cpu().numpy(), qt[f"{pre}{t}_sc"])
            check_vt(views[f"{pre}v_codes"][h].cpu().numpy(), views[f"{pre}v_scales"][h].cpu().numpy(),
                     qt[f"{pre}v_codes"], qt[f"{pre}v_sc"])
    sample = [i for i in qblocks if i not in rows]
    Oref = tiered_attention_head(Qh, Kh, Vh, rt, qt, cfg.low, cfg.block_q, cfg.block_k,
                                 cfg.p_offset_log2, rt["scale"], False, sample, threads=4,
                                 key_pack=cfg.key_pack)
    return assert_out_close(to64(O[0, h].cpu()), Oref, f"{cfg.name} head {h}")


@pytest.mark.parametrize("name", ["480p", "sweep0", "sweep30", "sweep50", "sweep70", "sweep90", "720p",
                                  "480p-price", "480p-entropy", "480p-fg"])
def test_fullsize_sampled_parity(cuda_ok, name):
    cfg, Q, K, V, views, O = _run_full(name)
    nqb = cfg.n_qb
    qblocks = [0, nqb // 2, nqb - 1]
    for h in (0, cfg.H - 1):
        _check_head(cfg, Q, K, V, views, O, h, qblocks)
    # every output row of every head is finite
    assert torch.isfinite(O.float()).all()
