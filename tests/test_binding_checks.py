"""The Python binding's operand checks: the C ABI takes bare pointers, so the
binding refuses, before any library call, tensors that would make a kernel
read the wrong memory (host tensors passed as device operands, another
dtype, storage shorter than the layout the parameters describe).  Every case
here raises on the host; no GPU is needed."""

import pytest
import torch

import precision_attention_video_b200 as pav
from precision_attention_video_b200 import binding as B


def _params(**kw):
    base = dict(B=1, H=2, N=100, d=64, block_q=64, block_k=64, low=1, tau=(0.6, 0.9),
                p_offset_log2=8)
    base.update(kw)
    return pav.make_params(**base)


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_span_follows_the_strides():
    p = _params()
    assert B._span(p) == 2 * 100 * 64                       # contiguous [1, 2, 100, 64]
    # heads interleaved per token ([B, N, H, d] storage): the same elements
    q = _params(strides=(100 * 2 * 64, 64, 2 * 64))
    assert B._span(q) == 2 * 100 * 64
    # padded rows: the last row still ends at its d-th element
    r = _params(B=2, strides=(2 * 100 * 72, 100 * 72, 72))
    assert B._span(r) == 2 * 2 * 100 * 72 - (72 - 64)


def test_host_tensors_are_refused_as_device_operands():
    p = _params()
    Q = _bf16(1, 2, 100, 64)
    ws = torch.zeros(pav.workspace_bytes(p), dtype=torch.uint8)
    for call in (lambda: pav.plan(p, Q, Q, Q, ws), lambda: pav.prep(p, Q, Q, Q, ws),
                 lambda: pav.forward(p, Q, Q, Q, ws, Q), lambda: pav.route(p, ws),
                 lambda: pav.get_status(ws),
                 lambda: pav.route_noalloc(p, Q, Q, Q, ws, ws, ws)):
        with pytest.raises(ValueError, match="expected a CUDA tensor"):
            call()


def test_layer_from_host_checks_its_host_buffers_first():
    p = _params()
    good = _bf16(1, 2, 100, 64)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(TypeError, match="Kh: expected torch.bfloat16"):
        pav.layer_from_host(p, good, good.float(), good, good, None, None, None, None, ws)
    with pytest.raises(ValueError, match="Oh: 12799 elements"):
        pav.layer_from_host(p, good, good, good, good.flatten()[1:], None, None, None, None, ws)
    # host buffers pass; the first device buffer is the next to be refused
    with pytest.raises(ValueError, match="Qd: expected a CUDA tensor"):
        pav.layer_from_host(p, good, good, good, good, good, good, good, good, ws)


def test_operand_checks_dtype_storage_and_kind():
    t = _bf16(2, 100, 64)
    n = t.numel()
    assert B._operand("X", t, cuda=False, dtype=torch.bfloat16, need=n) == t.data_ptr()
    with pytest.raises(TypeError, match="X: expected torch.bfloat16, got torch.float16"):
        B._operand("X", t.half(), cuda=False, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="expected a torch.Tensor"):
        B._operand("X", [0.0] * n, cuda=False)
    # storage counts from the view's first element: a view that starts one
    # row in has one row less behind it, whatever its own shape says
    v = t.view(-1, 64)[1:]
    assert B._elems_after(v) == n - 64
    with pytest.raises(ValueError, match="needs 12800"):
        B._operand("X", v, cuda=False, need=n)
    # a strided view reaches as far as its storage does
    w = t.view(1, 100, 2, 64).permute(0, 2, 1, 3)
    assert B._operand("X", w, cuda=False, need=n) == t.data_ptr()


def test_plan_views_wants_a_byte_workspace():
    p = _params()
    with pytest.raises(TypeError, match="ws: expected torch.uint8"):
        pav.plan_views(p, torch.zeros(8, dtype=torch.float32))
