"""The router entry point that allocates nothing.

tiered_attn_route_noalloc serves callers that cannot allocate device memory
(code inside a host framework that owns the GPU's memory, or a latency-critical
path where cudaMalloc would synchronise the device): its intermediates live in
a fixed array inside the library.  It must produce the same tier map, row
counts and row lists as tiered_attn_plan with the same params, for every
router, and keep doing so on back-to-back calls that reuse the array.  This
file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import inputs

pytestmark = pytest.mark.gpu


CASES = [
    ("tiny", {}),                                            # mass router, FP8
    ("small", {}),                                           # 128 x 64 tiles
    ("480p", {"H": 2, "grid": (3, 10, 21)}),                 # ragged N = 630, NVFP4
    ("720p", {"H": 2, "grid": (3, 9, 20)}),                  # ragged N = 540, four tiers
    ("480p-price", {"H": 2, "grid": (3, 10, 21), "price": 0.028}),   # price router
    ("small", {"H": 3, "router": 1, "price": 0.002}),        # price router, FP8 tiers
    ("480p", {"H": 2, "grid": (3, 10, 21), "router": 2, "kappa": 0.5}),  # entropy router
    ("720p", {"H": 2, "grid": (3, 9, 20), "router": 2, "kappa": 1.0}),   # entropy, four tiers
    ("480p-fg", {"H": 2, "grid": (3, 10, 21)}),              # 32-key blocks, ragged
    ("480p-fg", {"H": 1, "grid": (4, 32, 72)}),              # 288 32-key blocks a row (CTA-a-row router)
]


@pytest.mark.parametrize("name,over", CASES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(CASES)])
def test_noalloc_router_matches_plan_twice(cuda_ok, name, over):
    import precision_attention_video_b200 as pav
    cfg, Q, K, V = inputs(name, **over)
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
        c = cnt.cpu().numpy()
        assert (c.sum(axis=-1) == cfg.n_kb).all(), f"call {call}: counts do not cover every block"
        np.testing.assert_array_equal(tmap.cpu().numpy(), want_t, err_msg=f"call {call}")
        np.testing.assert_array_equal(c, want_c, err_msg=f"call {call}")
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
