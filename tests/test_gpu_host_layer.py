"""The end-to-end entry point tiered_attn_layer_from_host (host buffers in,
host buffer out; the layer runs in chunks of heads whose copies overlap the
kernels) gives bit for bit the output of plan + forward on device-resident
inputs, with a clean status."""

import pytest
import torch

from gpu_helpers import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [("small", {}), ("480p", {"grid": (3, 10, 21), "H": 5}),
                                       ("tiny", {"H": 1})])
def test_layer_from_host_matches_device_path(cuda_ok, name, over):
    import precision_attention_video_b200 as pav
    cfg, Q, K, V = inputs(name, **over)
    dev = torch.device("cuda:0")
    p = pav.params_for(cfg)
    # device path
    Qd, Kd, Vd = (x.to(dev) for x in (Q, K, V))
    ws = pav.alloc_workspace(p, dev)
    O = torch.empty_like(Qd)
    pav.plan(p, Qd, Kd, Vd, ws)
    pav.forward(p, Qd, Kd, Vd, ws, O)
    torch.cuda.synchronize()
    assert pav.get_status(ws) == 0
    # host path, fresh device buffers and workspace, run twice
    Qh, Kh, Vh = (x.pin_memory() for x in (Q, K, V))
    Oh = torch.empty_like(Q).pin_memory()
    Qd2, Kd2, Vd2, Od2 = (torch.empty_like(Qd) for _ in range(4))
    ws2 = pav.alloc_workspace(p, dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(2):
        Oh.zero_()
        pav.layer_from_host(p, Qh, Kh, Vh, Oh, Qd2, Kd2, Vd2, Od2, ws2, stream)
        torch.cuda.synchronize()
        assert pav.get_status(ws2) == 0
        assert torch.equal(Oh, O.cpu())
