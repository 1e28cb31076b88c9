"""Device-side failure detection without a GPU fault.

The test hook TA_DEBUG_DROP_FIRST_K makes the attention producer skip the first
K tile load, so the MMA issuer's bounded wait runs out (~1 s).  The kernel must
then report TA_ERR_TIMEOUT through the workspace status word, release its TMEM
and return; the context stays usable for the next call.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import assert_out_close, inputs, oracle_head, to64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_ok):
    import precision_attention_video_b200 as pav
    cfg, Q, K, V = inputs("tiny")
    dev = torch.device("cuda:0")
    Qd, Kd, Vd = (x.to(dev) for x in (Q, K, V))
    p = pav.params_for(cfg, debug_flags=pav.TA_DEBUG_DROP_FIRST_K)
    ws = pav.alloc_workspace(p, dev)
    O = torch.zeros_like(Qd)
    pav.plan(p, Qd, Kd, Vd, ws)
    pav.forward(p, Qd, Kd, Vd, ws, O)
    assert pav.get_status(ws) == pav.TA_ERR_TIMEOUT
    st = pav.plan_views(p, ws)["status"].cpu().numpy()
    assert st[1] in (1, 2, 3, 4, 5, 6, 7, 8)        # the wait site that ran out
    # a normal call afterwards works
    q = pav.params_for(cfg)
    pav.plan(q, Qd, Kd, Vd, ws)
    pav.forward(q, Qd, Kd, Vd, ws, O)
    assert pav.get_status(ws) == pav.TA_OK
    _, _, Oref = oracle_head(cfg, Q, K, V, 0, 0)
    assert_out_close(to64(O[0, 0].cpu()), Oref, "after timeout")
