"""Host-side logic of the benchmark: the algorithmic FLOP count per tier that
the roofline line divides by, checked against a hand count on a small plan,
and the summary of the clock samples taken during the timed region (median
SM clock, throttle reasons) that decides whether a run is kept."""

import importlib.util
import os

import numpy as np

from latent_gen import get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_flops_by_tier():
    bench = _bench()
    # N = 300 tokens in 128 x 128 tiles: blocks of 128, 128 and 44 rows / keys
    cfg = get_config("480p").with_(H=1, grid=(1, 3, 100), low=3, tau=(0.5, 0.7, 0.9))
    assert cfg.N == 300 and cfg.n_qb == 3 and cfg.n_kb == 3
    # one head; per query block: counts (full, res, low, skip) and list order
    counts = np.array([[[1, 1, 1, 0], [2, 0, 0, 1], [1, 0, 1, 1]]], dtype=np.int32)
    lists = np.array([[[0, 2, 1], [1, 2, 0], [2, 0, 1]]], dtype=np.int32)
    full, res, low, skip = bench.algorithmic_attn_flops(cfg, counts, lists)
    d = 128
    q = [128, 128, 44]
    k = [128, 128, 44]
    want_full = 4 * d * (q[0] * k[0] + q[1] * (k[1] + k[2]) + q[2] * k[2])
    want_res = 3 * 4 * d * (q[0] * k[2])
    want_low = 4 * d * (q[0] * k[1] + q[2] * k[0])
    want_skip = 4 * d * (q[1] * 1 + q[2] * 1)
    assert (full, res, low, skip) == (want_full, want_res, want_low, want_skip)


def test_clock_summary_from_nvidia_smi_lines():
    # lines as `nvidia-smi --query-gpu=... --format=csv,noheader,nounits` prints them:
    # index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
    # hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    bench = _bench()
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 612.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1845, 1965, 998.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 990.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",   # unreadable sample
        "garbled",
    ]
    s = cs.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1900.0            # median of 1965, 1845, 1900
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    cs.lines.append("0, 1200, 1965, 700.0, 0x0000000000000048, Active, Active, Not Active, Not Active")
    assert bench.ClockSampler.summary(cs)["reasons"] == ["hw_slowdown", "hw_thermal_slowdown",
                                                         "sw_power_cap"]
    cs.lines = []
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_bf16_peak_follows_the_sampled_clock():
    # burst peak when the timed region ran at the maximum SM clock with no
    # power cap; sustained peak otherwise (clock sank, or power-capped)
    bench = _bench()
    peaks = {"bf16_tflops": 1606.7, "bf16_tflops_sustained": 1365.0}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.bf16_peak(peaks, full)[0] == 1606.7
    assert "burst" in bench.bf16_peak(peaks, full)[1]
    capped = dict(full, reasons=["sw_power_cap"])
    assert bench.bf16_peak(peaks, capped)[0] == 1365.0
    slow = dict(full, sm_mhz=1305.0)
    assert bench.bf16_peak(peaks, slow)[0] == 1365.0
    none = {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}
    assert "sustained" in bench.bf16_peak(peaks, none)[1]


def test_kernel_named_in_the_roofline_follows_the_dispatch():
    # the two-group kernel for d = 128 with 128-query blocks and 128- or
    # 32-key blocks, except residual layers tiered by thresholds; the 16-warp
    # kernel for the other shapes (FP8 natively at every shape)
    from latent_gen import get_config
    want = {"480p": "attn2_kernel<LM_NVFP4, 128>", "480p-fg": "attn2_kernel<LM_NVFP4, 32>",
            "480p-price": "attn2_kernel<LM_NVFP4_RES, 128>", "sweep70": "attn2_kernel<LM_FP8, 128>",
            "720p": "attn_kernel<128, 128, LM_NVFP4_RES>", "small": "attn_kernel<64, 64, LM_FP8>",
            "tiny": "attn_kernel<64, 64, LM_FP8>"}
    bench = _bench()
    for name, kernel in want.items():
        assert bench.attn_kernel_name(get_config(name)) == kernel, name
    assert bench.attn_kernel_name(get_config("sweep70").with_(block_q=64)) == "attn_kernel<128, 128, LM_FP8>"


def test_traffic_figure_is_tied_to_the_kernel_sources():
    # the recorded DRAM traffic belongs to the sources it was captured on
    # (the bench line reports it only while the hash matches); the hash is
    # stable across calls and covers the kernel file, its headers and its
    # argument struct
    bench = _bench()
    h = bench.attn_source_sha1()
    assert len(h) == 40 and h == bench.attn_source_sha1()
    assert bench.ATTN_TRAFFIC["bytes_per_launch"] > 0 and len(bench.ATTN_TRAFFIC["source_sha1"]) == 40
