"""Pins of plan reuse across timesteps (oracle/route.py, reuse_plan): a plan
made on one timestep's inputs, with the block means and low-precision copies
of the current step.  On identical inputs it is the fresh plan; a plan that
keeps every tile in bf16 gives dense attention of the current step whatever
step it was made on; and on a slowly changing sequence the reused plan's
output stays close to the fresh plan's."""

import numpy as np

import oracle
from latent_gen import get_config
from latent_gen.generator import make_qkv_steps
from oracle import quant as Qz
from oracle import route as R
from oracle.attention import tiered_attention_head


def _heads(seq, h=0):
    return [tuple(x[0, h].double().numpy() for x in step) for step in seq]


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_steps_are_correlated_and_keep_the_marginals():
    cfg = get_config("480p").with_(H=1, grid=(2, 8, 16))
    seq = make_qkv_steps(cfg, 3, rho=0.9)
    q0, q1, q2 = (s[0].float().flatten() for s in seq)
    c = float(np.corrcoef(q0.numpy(), q1.numpy())[0, 1])
    assert 0.85 < c < 0.95
    assert float(np.corrcoef(q0.numpy(), q2.numpy())[0, 1]) < c
    assert abs(float(q2.std()) / float(q0.std()) - 1.0) < 0.05


def test_reuse_on_the_same_inputs_is_the_fresh_plan():
    cfg = get_config("480p").with_(H=1, grid=(3, 10, 21))
    (Qh, Kh, Vh), = _heads(make_qkv_steps(cfg, 1, rho=1.0))
    rt = R.route_head(Qh, Kh, Vh, cfg.tau, cfg.block_q, cfg.block_k)
    ru = R.reuse_plan(rt, Qh, Kh, Vh, cfg.block_q, cfg.block_k)
    for k in ("tiers", "counts", "lists", "kbar_b", "vbar_b", "n_k", "M"):
        np.testing.assert_array_equal(np.asarray(ru[k]), np.asarray(rt[k]))


def test_all_full_plan_reused_is_dense_attention_of_the_current_step():
    cfg = get_config("480p").with_(H=1, grid=(2, 8, 20), tau=(2.0, 2.0))
    steps = _heads(make_qkv_steps(cfg, 3, rho=0.8))
    Q0, K0, V0 = steps[0]
    rt0 = R.route_head(Q0, K0, V0, cfg.tau, cfg.block_q, cfg.block_k)
    assert (rt0["tiers"] == R.TIER_FULL).all()
    Q2, K2, V2 = steps[2]
    ru = R.reuse_plan(rt0, Q2, K2, V2, cfg.block_q, cfg.block_k)
    qt = Qz.quantize_head(Q2, K2, V2, cfg.low, cfg.block_q, cfg.block_k)
    O = tiered_attention_head(Q2, K2, V2, ru, qt, cfg.low, cfg.block_q, cfg.block_k,
                              cfg.p_offset_log2, ru["scale"], exact=True)
    assert _rel(O, oracle.dense_attention(Q2, K2, V2)) <= 1e-12


def test_reused_plan_stays_close_on_a_slow_sequence():
    cfg = get_config("480p").with_(H=1, grid=(3, 10, 21))
    steps = _heads(make_qkv_steps(cfg, 2, rho=0.98))
    Q0, K0, V0 = steps[0]
    Q1, K1, V1 = steps[1]
    rt0 = R.route_head(Q0, K0, V0, cfg.tau, cfg.block_q, cfg.block_k)
    rt1 = R.route_head(Q1, K1, V1, cfg.tau, cfg.block_q, cfg.block_k)
    qt = Qz.quantize_head(Q1, K1, V1, cfg.low, cfg.block_q, cfg.block_k)
    ru = R.reuse_plan(rt0, Q1, K1, V1, cfg.block_q, cfg.block_k)
    args = (cfg.low, cfg.block_q, cfg.block_k, cfg.p_offset_log2, rt1["scale"], True)
    O_fresh = tiered_attention_head(Q1, K1, V1, rt1, qt, *args)
    O_reuse = tiered_attention_head(Q1, K1, V1, ru, qt, *args)
    D = oracle.dense_attention(Q1, K1, V1)
    # the tier maps mostly agree, and the reused plan's error against dense
    # attention stays of the order of the fresh plan's
    assert (rt0["tiers"] == rt1["tiers"]).mean() > 0.8
    assert _rel(O_reuse, D) <= 2.0 * _rel(O_fresh, D) + 1e-3
