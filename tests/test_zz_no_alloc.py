"""The router entry point that allocates nothing.

tiered_attn_route_noalloc serves callers that cannot allocate device memory
(code inside a host framework that owns the GPU's memory, or a latency-critical
path where cudaMalloc would synchronise the device): its intermediates live in
a fixed array inside the library.  It must produce the same tier map, row
counts and row lists as tiered_attn_plan, and keep doing so on back-to-back
calls that reuse the array.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_noalloc_router_matches_plan_twice(cuda_ok, name):
    import precision_attention_video_b200 as pav
    cfg, Q, K, V = inputs(name)
    dev = torch.device("cuda:0")
    Qd, Kd, Vd = (x.to(dev) for x in (Q, K, V))
    p = pav.params_for(cfg)
    ws = pav.alloc_workspace(p, dev)
    pav.plan(p, Qd, Kd, Vd, ws)
    views = pav.plan_views(p, ws)
    want_t = views["tier_map"].cpu().numpy()
    want_c = views["row_counts"].cpu().numpy()
    want_l = views["row_lists"].cpu().numpy()
    BH = cfg.B * cfg.H
    for call in range(2):
        tmap = torch.full((BH, cfg.n_qb, cfg.n_kb), 255, dtype=torch.uint8, device=dev)
        cnt = torch.full((BH, cfg.n_qb, 4), -1, dtype=torch.int32, device=dev)
        lst = torch.full((BH, cfg.n_qb, cfg.n_kb), -1, dtype=torch.int32, device=dev)
        pav.route_noalloc(p, Qd, Kd, Vd, tmap, cnt, lst)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(tmap.cpu().numpy(), want_t, err_msg=f"call {call}")
        np.testing.assert_array_equal(cnt.cpu().numpy(), want_c, err_msg=f"call {call}")
        np.testing.assert_array_equal(lst.cpu().numpy(), want_l, err_msg=f"call {call}")


def test_noalloc_router_rejects_problems_beyond_its_scratch(cuda_ok):
    import precision_attention_video_b200 as pav
    from latent_gen import get_config
    cfg = get_config("480p")   # intermediates of about 68 MB > the fixed 16 MB
    p = pav.params_for(cfg)
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda:0")
    out = torch.empty(16, dtype=torch.int32, device="cuda:0")
    with pytest.raises(pav.TieredAttnError) as e:
        pav.route_noalloc(p, x, x, x, out, out, out)
    assert e.value.code == pav.TA_ERR_WORKSPACE
