"""Shared machinery of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare them."""

from __future__ import annotations

from functools import lru_cache

import numpy as np
import torch

import oracle
from latent_gen import get_config, make_qkv
from oracle import quant as Qz
from oracle import route as Rt

# Output bar (floating point): relative L2 <= 1e-2 and max-abs <= 2e-2 against
# the oracle fed the same quantised operands.
REL_L2 = 1e-2
MAX_ABS = 2e-2


@lru_cache(maxsize=4)
def inputs(name: str, **over):
    cfg = get_config(name)
    if over:
        cfg = cfg.with_(**dict(over))
    Q, K, V = make_qkv(cfg)
    return cfg, Q, K, V


def to64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float64).numpy()


def run_gpu(cfg, Q, K, V, forward=True, **param_over):
    import precision_attention_video_b200 as pav
    p = pav.params_for(cfg, **param_over)
    dev = torch.device("cuda:0")
    Qd, Kd, Vd = (x.to(dev) for x in (Q, K, V))
    ws = pav.alloc_workspace(p, dev)
    pav.plan(p, Qd, Kd, Vd, ws)
    O = None
    if forward:
        O = torch.empty_like(Qd)
        pav.forward(p, Qd, Kd, Vd, ws, O)
    torch.cuda.synchronize()
    st = pav.get_status(ws)
    views = {k: v.cpu() for k, v in pav.plan_views(p, ws).items()}
    return p, views, (O.cpu() if O is not None else None), st


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """[..., n/2] bytes -> [..., n] codes (element 2c in the low nibble)."""
    lo = packed & 0x0F
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)


def router_kwargs(cfg, low=None):
    """route_head keywords of the workload's router (mass thresholds or price)."""
    return {"router": getattr(cfg, "router", 0), "price": getattr(cfg, "price", 0.0),
            "low": cfg.low if low is None else low, "kappa": getattr(cfg, "kappa", 1.0),
            "tier_cost": getattr(cfg, "tier_cost", None)}


def oracle_head(cfg, Q, K, V, b, h, qblocks=None, exact=False, tau=None, low=None,
                keep_diag=True):
    Qh, Kh, Vh = to64(Q[b, h]), to64(K[b, h]), to64(V[b, h])
    tau = cfg.tau if tau is None else tau
    low = cfg.low if low is None else low
    rt = Rt.route_head(Qh, Kh, Vh, tau, cfg.block_q, cfg.block_k, keep_diag_full=keep_diag,
                       **router_kwargs(cfg, low))
    qt = Qz.quantize_head(Qh, Kh, Vh, low, cfg.block_q, cfg.block_k)
    O = None
    if qblocks != []:
        O = oracle.tiered_attention_head(Qh, Kh, Vh, rt, qt, low, cfg.block_q, cfg.block_k,
                                         cfg.p_offset_log2, rt["scale"], exact, qblocks,
                                         key_pack=cfg.key_pack)
    return rt, qt, O


def compare_tiers(gpu_tiers: np.ndarray, rt: dict):
    """Tier map equal except on oracle-flagged tiles; returns (n_diff, rows that differ)."""
    diff = gpu_tiers != rt["tiers"]
    bad = diff & ~rt["flags"]
    assert not bad.any(), f"{int(bad.sum())} unflagged tier differences at {np.argwhere(bad)[:5]}"
    return int(diff.sum()), set(np.nonzero(diff.any(axis=1))[0].tolist())


def check_lists(tiers: np.ndarray, counts: np.ndarray, lists: np.ndarray, mass: np.ndarray):
    """Each row's list is a permutation grouped full, res, low, skip; within a
    tier ordered by (-M, j) of the router's (GPU) masses."""
    order = [3, 2, 1, 0]
    for i in range(tiers.shape[0]):
        pos = 0
        rank = np.lexsort((np.arange(tiers.shape[1]), -mass[i]))
        for q, t in enumerate(order):
            want = rank[tiers[i][rank] == t]
            assert counts[i, q] == len(want), (i, t)
            np.testing.assert_array_equal(lists[i, pos:pos + len(want)], want)
            pos += len(want)
        assert pos == tiers.shape[1]


def check_vt(gpu_codes_packed: np.ndarray, gpu_sc: np.ndarray, o_codes: np.ndarray,
             o_sc: np.ndarray):
    """GPU transposed NVFP4 V copy ([d, Np/2] packed, scales [Np/16, d]) equals
    the oracle's column copy ([Np16, d], scales [Np16/16, d]); the extra pitch
    tokens are zero."""
    vt = unpack_fp4(gpu_codes_packed).T
    n = o_codes.shape[0]
    np.testing.assert_array_equal(vt[:n], o_codes)
    assert not vt[n:].any()
    g = o_sc.shape[0]
    np.testing.assert_array_equal(gpu_sc[:g], o_sc)
    assert not gpu_sc[g:].any()


def out_errors(O_gpu: np.ndarray, O_ref: np.ndarray):
    m = ~np.isnan(O_ref[:, 0])
    a, r = O_gpu[m], O_ref[m]
    rel = np.linalg.norm(a - r) / np.linalg.norm(r)
    mx = np.abs(a - r).max()
    return float(rel), float(mx), int(m.sum())


def assert_out_close(O_gpu: np.ndarray, O_ref: np.ndarray, what: str = ""):
    rel, mx, n = out_errors(O_gpu, O_ref)
    assert n > 0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e} over {n} rows"
    return rel, mx
