"""The C ABI library: it loads, exports every symbol include/tiered_attn.h
declares, and validates arguments on the host (no GPU needed: every case here
returns before any CUDA call)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tiered_attn_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def pav():
    import precision_attention_video_b200 as m
    return m


def test_header_declares_entry_points():
    names = _declared()
    for must in ("tiered_attn_plan", "tiered_attn_forward", "tiered_attn_workspace_bytes",
                 "tiered_attn_plan_views", "tiered_attn_get_status"):
        assert must in names


def test_library_exports_every_declared_symbol(pav):
    lib = ctypes.CDLL(pav.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(pav):
    assert pav.status_string(0) == "ok"
    assert "timed out" in pav.status_string(-5)
    assert pav.version() >= 100


def _params(pav, **kw):
    base = dict(B=1, H=2, N=1000, d=64, block_q=64, block_k=64, low=1, tau=(0.6, 0.9),
                p_offset_log2=8)
    base.update(kw)
    return pav.make_params(**base)


def test_workspace_bytes_and_validation(pav):
    p = _params(pav)
    n = pav.workspace_bytes(p)
    assert n > 0 and n % 256 == 0
    bigger = pav.workspace_bytes(_params(pav, N=4000))
    assert bigger > n
    assert pav.workspace_bytes(_params(pav, low=2)) > 0
    assert pav.workspace_bytes(_params(pav, low=3, tau=(0.5, 0.6, 0.8))) > pav.workspace_bytes(_params(pav, low=2))
    bad = [
        dict(d=96), dict(block_q=32), dict(N=0), dict(low=7), dict(tau=(0.9, 0.6)),
        dict(low=3), dict(low=0), dict(p_offset_log2=40), dict(N=200000),
        dict(strides=(2 * 1000 * 64, 1000 * 64, 60)),
        dict(router=3), dict(router=-1), dict(router=1, price=-1e-3),
        dict(router=1, price=float("nan")), dict(router=1, price=float("inf")),
        dict(router=2, retention=0.0), dict(router=2, retention=-1.0),
        dict(router=2, retention=float("nan")),
    ]
    for kw in bad:
        assert pav.workspace_bytes(_params(pav, **kw)) == 0, kw
    # the price router adds its block statistics to the workspace; the
    # entropy router needs none
    assert pav.workspace_bytes(_params(pav, router=1, price=1e-3)) > n
    assert pav.workspace_bytes(_params(pav, router=2, retention=0.5)) == n


def test_shape_limits_at_their_edges(pav):
    ws = pav.workspace_bytes
    fg = dict(d=128, block_q=128, block_k=32, low=2, tau=(0.6, 0.9))   # NVFP4
    # 32-key blocks: d = 128, 128-query blocks, bf16 / NVFP4 / NVFP4 + residual
    assert ws(_params(pav, **fg)) > 0
    assert ws(_params(pav, **dict(fg, low=0, tau=(0.9,)))) > 0
    assert ws(_params(pav, **dict(fg, low=3, tau=(0.5, 0.6, 0.8)))) > 0
    assert ws(_params(pav, **dict(fg, low=1))) == 0        # FP8
    assert ws(_params(pav, **dict(fg, d=64))) == 0
    assert ws(_params(pav, **dict(fg, block_q=64))) == 0
    # the router sorts at most 1024 key blocks a row: N up to 1024 blocks,
    # the last one ragged or whole, and not one token more
    for bk in (32, 64, 128):
        kw = dict(fg, block_k=bk)
        assert ws(_params(pav, **dict(kw, N=1024 * bk))) > 0, bk
        assert ws(_params(pav, **dict(kw, N=1023 * bk + 1))) > 0, bk
        assert ws(_params(pav, **dict(kw, N=1024 * bk + 1))) == 0, bk
    # one CTA row per (batch, head): B * H <= 65535
    assert ws(_params(pav, B=1, H=65535, N=64)) > 0
    assert ws(_params(pav, B=3, H=21845, N=64)) > 0
    assert ws(_params(pav, B=2, H=32768, N=64)) == 0
    # P' offsets 2^0 .. 2^15
    assert ws(_params(pav, p_offset_log2=0)) > 0
    assert ws(_params(pav, p_offset_log2=15)) > 0
    assert ws(_params(pav, p_offset_log2=16)) == 0
    assert ws(_params(pav, p_offset_log2=-1)) == 0


def test_calls_reject_bad_arguments_before_launch(pav):
    lib = pav.binding.lib() if hasattr(pav, "binding") else None
    from precision_attention_video_b200 import binding as B
    p = _params(pav)
    need = pav.workspace_bytes(p)
    # null tensors
    st = B.lib().tiered_attn_plan(ctypes.byref(p), None, None, None, None, 0, None)
    assert st == pav.TA_ERR_INVALID_ARG
    # misaligned tensor pointer
    st = B.lib().tiered_attn_plan(ctypes.byref(p), 0x1008, 0x1000, 0x1000, 0x10000, need, None)
    assert st == pav.TA_ERR_INVALID_ARG
    # misaligned workspace
    st = B.lib().tiered_attn_plan(ctypes.byref(p), 0x1000, 0x1000, 0x1000, 0x10010, need, None)
    assert st == pav.TA_ERR_INVALID_ARG
    # workspace too small
    st = B.lib().tiered_attn_plan(ctypes.byref(p), 0x1000, 0x1000, 0x1000, 0x10000, need - 256, None)
    assert st == pav.TA_ERR_WORKSPACE
    st = B.lib().tiered_attn_forward(ctypes.byref(p), 0x1000, 0x1000, 0x1000, 0x10000, need - 256,
                                     0x2000, None)
    assert st == pav.TA_ERR_WORKSPACE
    # invalid params
    q = _params(pav, d=96)
    assert B.lib().tiered_attn_forward(ctypes.byref(q), 0x1000, 0x1000, 0x1000, 0x10000, need,
                                       0x2000, None) == pav.TA_ERR_UNSUPPORTED
    assert B.lib().tiered_attn_plan_views(ctypes.byref(p), None, None) == pav.TA_ERR_INVALID_ARG
    assert B.lib().tiered_attn_get_status(None, None) == pav.TA_ERR_INVALID_ARG
    del lib


def test_plan_views_offsets_inside_workspace(pav):
    from precision_attention_video_b200 import binding as B
    for low, tau in ((1, (0.6, 0.9)), (2, (0.6, 0.9)), (3, (0.5, 0.675, 0.85)), (0, (0.6,))):
        p = _params(pav, low=low, tau=tau, d=128, block_q=128, block_k=128)
        need = pav.workspace_bytes(p)
        base = 1 << 20
        v = B.ta_plan_views()
        assert B.lib().tiered_attn_plan_views(ctypes.byref(p), base, ctypes.byref(v)) == 0
        assert v.status == base
        ptrs = [getattr(v, n) for n, _ in B.ta_plan_views._fields_ if getattr(v, n)]
        assert all(base <= x < base + need for x in ptrs)
        assert all((x - base) % 256 == 0 for x in ptrs)
        assert (v.q_codes is not None) == (low != 0)
        assert (v.rq_codes is not None) == (low == 3)
