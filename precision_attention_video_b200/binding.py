"""ctypes binding of libtiered_attn.so (the C ABI declared in include/tiered_attn.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  If the
shared library is missing this module raises at import time; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtiered_attn.so")

TA_OK = 0
TA_ERR_INVALID_ARG = -1
TA_ERR_UNSUPPORTED = -2
TA_ERR_WORKSPACE = -3
TA_ERR_CUDA = -4
TA_ERR_TIMEOUT = -5

TA_LOW_NONE, TA_LOW_FP8_E4M3, TA_LOW_NVFP4, TA_LOW_NVFP4_RES = 0, 1, 2, 3
TA_TIER_SKIP, TA_TIER_LOW, TA_TIER_RES, TA_TIER_FULL = 0, 1, 2, 3
TA_DEBUG_DROP_FIRST_K = 1


class ta_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
        ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("low", ctypes.c_int32), ("n_thresholds", ctypes.c_int32),
        ("tau", ctypes.c_double * 3),
        ("keep_diag_full", ctypes.c_int32), ("p_offset_log2", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("debug_flags", ctypes.c_int32),
        ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64), ("stride_n", ctypes.c_int64),
        ("router", ctypes.c_int32), ("price", ctypes.c_double), ("retention", ctypes.c_double),
        ("tier_cost", ctypes.c_double * 4),
    ]


_VIEW_FIELDS = [
    "status", "qbar", "kbar", "kbar_b", "vbar_b", "n_k", "logits", "mass", "tier_map",
    "row_counts", "row_lists", "q_codes", "k_codes", "v_codes", "q_scales", "k_scales",
    "v_scales", "rq_codes", "rk_codes", "rv_codes", "rq_scales", "rk_scales", "rv_scales",
    "dq", "dk", "dv", "drq", "drk", "drv", "kvar", "spread", "qvar",
]


class ta_plan_views(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _VIEW_FIELDS]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m precision_attention_video_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(ta_params)
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    sigs = {
        "tiered_attn_workspace_bytes": (sz, [P]),
        "tiered_attn_plan": (st, [P, vp, vp, vp, vp, sz, vp]),
        "tiered_attn_forward": (st, [P, vp, vp, vp, vp, sz, vp, vp]),
        "tiered_attn_layer_from_host": (st, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "tiered_attn_plan_views": (st, [P, vp, ctypes.POINTER(ta_plan_views)]),
        "tiered_attn_get_status": (st, [vp, vp]),
        "tiered_attn_prep": (st, [P, vp, vp, vp, vp, sz, vp]),
        "tiered_attn_route": (st, [P, vp, sz, vp]),
        "tiered_attn_route_noalloc": (st, [P, vp, vp, vp, vp, vp, vp, vp]),
        "tiered_attn_status_string": (ctypes.c_char_p, [st]),
        "tiered_attn_version": (ctypes.c_int32, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; loaded on first use, so that the package (and its
    build module) imports before the library exists.  Every call into the
    compute path goes through here and raises if the library is missing."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def status_string(code: int) -> str:
    return lib().tiered_attn_status_string(code).decode()


class TieredAttnError(RuntimeError):
    def __init__(self, call: str, code: int):
        super().__init__(f"{call}: {status_string(code)} ({code})")
        self.code = code


def _check(call: str, code: int) -> None:
    if code != TA_OK:
        raise TieredAttnError(call, code)


def _span(p: ta_params) -> int:
    """Elements from the first element of a [B, H, N, d] operand with p's
    strides to one past the last one the library reads or writes."""
    return (p.B - 1) * p.stride_b + (p.H - 1) * p.stride_h + (p.N - 1) * p.stride_n + p.d


def _elems_after(t: torch.Tensor) -> int:
    """Elements of t's storage from t's first element on."""
    return t.untyped_storage().nbytes() // t.element_size() - t.storage_offset()


def _operand(name: str, t, *, cuda: bool = True, dtype=None, need: int = 0) -> int:
    """t's data pointer, after the checks that the C ABI cannot make on a bare
    pointer: a CUDA tensor on the current device (the library launches there)
    or, with cuda=False, a host tensor; of `dtype`; with at least `need`
    elements of storage from its first element on."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if cuda:
        if not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")
        cur = torch.cuda.current_device()
        if t.device.index != cur:
            raise ValueError(f"{name}: on {t.device}, but the library launches on the current "
                             f"device cuda:{cur}")
    elif t.device.type != "cpu":
        raise ValueError(f"{name}: expected a host tensor, got one on {t.device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if need and _elems_after(t) < need:
        raise ValueError(f"{name}: {_elems_after(t)} elements of storage from its first element, "
                         f"the layout of the parameters needs {need}")
    return t.data_ptr()


def _qkv(p: ta_params, Q, K, V, cuda: bool = True, names=("Q", "K", "V")):
    """Pointers of three bf16 [B, H, N, d] operands laid out by p's strides."""
    n = _span(p)
    return tuple(_operand(nm, t, cuda=cuda, dtype=torch.bfloat16, need=n)
                 for nm, t in zip(names, (Q, K, V)))


def _ws(ws) -> int:
    return _operand("ws", ws, dtype=torch.uint8)


def make_params(B: int, H: int, N: int, d: int, block_q: int, block_k: int, low: int,
                tau: Sequence[float], p_offset_log2: int, keep_diag_full: int = 1,
                softmax_scale: float = 0.0, debug_flags: int = 0,
                strides: Optional[Sequence[int]] = None, router: int = 0,
                price: float = 0.0, retention: float = 1.0,
                tier_cost: Sequence[float] = (0.0, 0.0, 0.0, 0.0)) -> ta_params:
    """ta_params for a [B, H, N, d] layout (contiguous unless ``strides`` = (sb, sh, sn))."""
    p = ta_params()
    p.B, p.H, p.N, p.d = B, H, N, d
    p.block_q, p.block_k, p.low = block_q, block_k, low
    p.n_thresholds = len(tau)
    for i, t in enumerate(tau):
        p.tau[i] = float(t)
    p.keep_diag_full, p.p_offset_log2 = keep_diag_full, p_offset_log2
    p.softmax_scale, p.debug_flags = softmax_scale, debug_flags
    sb, sh, sn = strides if strides is not None else (H * N * d, N * d, d)
    p.stride_b, p.stride_h, p.stride_n = sb, sh, sn
    p.router, p.price, p.retention = router, float(price), float(retention)
    for i in range(4):
        p.tier_cost[i] = float(tier_cost[i])   # by tier code; all zero: the library's defaults
    return p


def params_for(cfg, **overrides) -> ta_params:
    """ta_params of a ``latent_gen.Workload``."""
    kw = dict(B=cfg.B, H=cfg.H, N=cfg.N, d=cfg.d, block_q=cfg.block_q, block_k=cfg.block_k,
              low=cfg.low, tau=cfg.tau, p_offset_log2=cfg.p_offset_log2,
              keep_diag_full=cfg.keep_diag_full, router=getattr(cfg, "router", 0),
              price=getattr(cfg, "price", 0.0), retention=getattr(cfg, "kappa", 1.0),
              tier_cost=getattr(cfg, "tier_cost", (0.0, 0.0, 0.0, 0.0)))
    kw.update(overrides)
    return make_params(**kw)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def workspace_bytes(p: ta_params) -> int:
    return int(lib().tiered_attn_workspace_bytes(ctypes.byref(p)))


def alloc_workspace(p: ta_params, device="cuda") -> torch.Tensor:
    n = workspace_bytes(p)
    if n == 0:
        raise TieredAttnError("tiered_attn_workspace_bytes", TA_ERR_INVALID_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device)


def plan(p: ta_params, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, ws: torch.Tensor,
         stream=None) -> None:
    q, k, v = _qkv(p, Q, K, V)
    _check("tiered_attn_plan", lib().tiered_attn_plan(
        ctypes.byref(p), q, k, v, _ws(ws), ws.numel(), _stream(stream)))


def prep(p, Q, K, V, ws, stream=None) -> None:
    q, k, v = _qkv(p, Q, K, V)
    _check("tiered_attn_prep", lib().tiered_attn_prep(
        ctypes.byref(p), q, k, v, _ws(ws), ws.numel(), _stream(stream)))


def route(p, ws, stream=None) -> None:
    _check("tiered_attn_route", lib().tiered_attn_route(
        ctypes.byref(p), _ws(ws), ws.numel(), _stream(stream)))


def route_noalloc(p: ta_params, Q, K, V, tier_map, row_counts, row_lists, stream=None) -> None:
    """Tier map, row counts and row lists without any workspace: the router's
    intermediates live in the library's fixed device array (see the header).
    Operands must be CUDA tensors on the current device, Q, K, V bf16; their
    sizes are the caller's to get right, as in the C ABI (the library checks
    the problem against its scratch before reading any of them)."""
    q, k, v = (_operand(nm, t, dtype=torch.bfloat16) for nm, t in (("Q", Q), ("K", K), ("V", V)))
    _check("tiered_attn_route_noalloc", lib().tiered_attn_route_noalloc(
        ctypes.byref(p), q, k, v, _operand("tier_map", tier_map),
        _operand("row_counts", row_counts), _operand("row_lists", row_lists), _stream(stream)))


def forward(p: ta_params, Q, K, V, ws, O, stream=None) -> None:
    q, k, v = _qkv(p, Q, K, V)
    o = _operand("O", O, dtype=torch.bfloat16, need=_span(p))
    _check("tiered_attn_forward", lib().tiered_attn_forward(
        ctypes.byref(p), q, k, v, _ws(ws), ws.numel(), o, _stream(stream)))


def layer_from_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, Od, ws, stream=None) -> None:
    """One layer from host buffers: Qh, Kh, Vh, Oh host bf16 tensors (pinned
    for overlapped copies), Qd, Kd, Vd, Od device bf16 tensors of the same
    layout, all laid out by p's strides."""
    qh, kh, vh = _qkv(p, Qh, Kh, Vh, cuda=False, names=("Qh", "Kh", "Vh"))
    oh = _operand("Oh", Oh, cuda=False, dtype=torch.bfloat16, need=_span(p))
    qd, kd, vd = _qkv(p, Qd, Kd, Vd, names=("Qd", "Kd", "Vd"))
    od = _operand("Od", Od, dtype=torch.bfloat16, need=_span(p))
    _check("tiered_attn_layer_from_host", lib().tiered_attn_layer_from_host(
        ctypes.byref(p), qh, kh, vh, oh, qd, kd, vd, od, _ws(ws), ws.numel(), _stream(stream)))


def get_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib().tiered_attn_get_status(_ws(ws), _stream(stream)))


def plan_views(p: ta_params, ws: torch.Tensor) -> Dict[str, torch.Tensor]:
    """Typed tensor views of a planned workspace (no copies)."""
    v = ta_plan_views()
    if ws.dtype != torch.uint8:
        raise TypeError(f"ws: expected torch.uint8, got {ws.dtype}")
    _check("tiered_attn_plan_views", lib().tiered_attn_plan_views(
        ctypes.byref(p), ws.data_ptr(), ctypes.byref(v)))
    BH = p.B * p.H
    N, d = p.N, p.d
    nqb = -(-N // p.block_q)
    nkb = -(-N // p.block_k)
    Np = 32 * (-(-N // 32))
    u8, i32, f64, f32, b16 = torch.uint8, torch.int32, torch.float64, torch.float32, torch.bfloat16
    shapes = {
        "status": (i32, (4,)), "qbar": (f64, (BH, nqb, d)), "kbar": (f64, (BH, nkb, d)),
        "kbar_b": (b16, (BH, nkb, d)), "vbar_b": (b16, (BH, nkb, d)), "n_k": (i32, (nkb,)),
        "logits": (f64, (BH, nqb, nkb)), "mass": (f64, (BH, nqb, nkb)),
        "tier_map": (u8, (BH, nqb, nkb)), "row_counts": (i32, (BH, nqb, 4)),
        "row_lists": (i32, (BH, nqb, nkb)),
        "dq": (b16, (BH, N, d)), "dk": (b16, (BH, N, d)), "dv": (b16, (BH, N, d)),
        "drq": (b16, (BH, N, d)), "drk": (b16, (BH, N, d)), "drv": (b16, (BH, N, d)),
        "kvar": (f64, (BH, nkb, d)), "spread": (f64, (BH, nqb, nkb)), "qvar": (f64, (BH, nqb, d)),
    }
    if p.low == TA_LOW_FP8_E4M3:
        shapes.update({"q_codes": (u8, (BH, N, d)), "k_codes": (u8, (BH, N, d)),
                       "v_codes": (u8, (BH, N, d)), "q_scales": (f32, (BH, nqb)),
                       "k_scales": (f32, (BH, nkb)), "v_scales": (f32, (BH, nkb))})
    else:
        for pre in ("", "r"):
            shapes.update({pre + "q_codes": (u8, (BH, N, d // 2)), pre + "k_codes": (u8, (BH, N, d // 2)),
                           pre + "v_codes": (u8, (BH, d, Np // 2)),
                           pre + "q_scales": (u8, (BH, N, d // 16)),
                           pre + "k_scales": (u8, (BH, N, d // 16)),
                           pre + "v_scales": (u8, (BH, Np // 16, d))})
    base = ws.data_ptr()
    out = {}
    for name in _VIEW_FIELDS:
        ptr = getattr(v, name)
        if not ptr or name not in shapes:
            continue
        dt, shp = shapes[name]
        nbytes = math.prod(shp) * torch.empty((), dtype=dt).element_size()
        off = ptr - base
        out[name] = ws[off:off + nbytes].view(dt).view(shp)
    return out


def version() -> int:
    return int(lib().tiered_attn_version())
