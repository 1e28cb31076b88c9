"""Benchmark of the tiered-precision video-DiT attention layer on B200.

One step = one full attention layer of the 480p-video-like workload
(B=1, H=40, N=32760 tokens from a 21x30x52 latent grid, d=128, 128x128 tiles,
NVFP4 low tier, cumulative-mass thresholds 0.6 / 0.9): tiered_attn_plan
(pooling, quantisation, routing) followed by tiered_attn_forward, on inputs
already resident in HBM.  The metric is dense-equivalent attention TFLOPS,
4*B*H*N^2*d / (plan + forward time); ms per layer and the attention kernel's
fraction of tensor-pipe peak for the FLOPs it executes are reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With --gpus N > 1 (launched by torchrun) each rank runs an independent
replica of the layer on its own GPU (the heads of a layer need no exchange);
`value` is the work of all ranks divided by the slowest rank's time.
--impl reference times the CPU oracle (fp64, software FP8/NVFP4 rounding) on
the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from latent_gen import get_config, make_qkv  # noqa: E402

WORKLOAD = "480p"
METRIC = "dense-equiv attention TFLOPS & ms/layer @32760 tok; % tensor-pipe peak"
UNIT = "TFLOPS"
L2_BYTES = 126 * 2 ** 20

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one forward
# launch of the 480p-video-like layer, from the ncu capture of the two-group
# kernel (attn2_kernel<LM_NVFP4, 128>) on 8 heads of that layer, scaled to 40
# by heads (traffic grows with the (head, query block) rows); valid only for
# the kernel sources it was measured on and for that workload.
ATTN_TRAFFIC = {"source_sha1": "c6ce1c5746f83ed3fa1b162b3b4376714885727e", "bytes_per_launch": 1596980480}


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def bf16_peak(peaks, clocks):
    """The bf16 tensor peak that applies to this run: the burst figure (a
    short matmul at full clock) when the sampled SM clock stayed at its
    maximum with no power cap, else the sustained one (a seconds-long matmul
    whose clock sank under the power cap).  Returns (TFLOP/s, which)."""
    burst = float(peaks.get("bf16_tflops", 0.0) or 0.0)
    sustained = float(peaks.get("bf16_tflops_sustained", burst) or burst)
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    full_clock = sm is not None and mx and sm >= 0.97 * mx
    if burst and full_clock and "sw_power_cap" not in clocks.get("reasons", []):
        return burst, f"burst bf16_tflops (SM clock {sm:.0f} of {mx:.0f} MHz, no power cap)"
    return sustained, "sustained bf16_tflops_sustained (SM clock below max or power-capped)"


def attn_source_sha1():
    """Hash of the attention kernel's sources (the kernel and the headers it
    inlines): a traffic figure holds only for the code it was measured on."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "precision_attention_video_b200", "csrc")
    for name in ("ta_attn2.cu", "ta_attn_common.cuh", "ta_common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    # of the shared argument header, only the struct the kernel takes
    with open(os.path.join(csrc, "ta_kernels.cuh")) as f:
        hdr = f.read()
    start = hdr.index("struct AttnArgs {")
    h.update(hdr[start:hdr.index("};", start)].encode())
    return h.hexdigest()


def attn_kernel_name(cfg) -> str:
    """The forward kernel the library dispatches for a workload: the
    two-group kernel for d = 128 with 128-query blocks and 128- or 32-key
    blocks (except NVFP4 + residual layers tiered by thresholds), the 16-warp
    kernel otherwise."""
    lm = {0: "LM_IMAGE", 1: "LM_FP8", 2: "LM_NVFP4", 3: "LM_NVFP4_RES"}[cfg.low]
    two_group = (cfg.d == 128 and cfg.block_q == 128 and cfg.block_k in (32, 128)
                 and not (cfg.low == 3 and cfg.block_k == 128 and getattr(cfg, "router", 0) != 1))
    if two_group:
        return f"attn2_kernel<{lm}, {cfg.block_k}>"
    return f"attn_kernel<{cfg.d}, {cfg.block_k}, {lm}>"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        self.first = threading.Event()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # nvidia-smi takes a while to start: the timed region begins only
            # once it is sampling, so that the samples fall inside it
            self.first.wait(timeout=5.0)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())
            self.first.set()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def algorithmic_attn_flops(cfg, counts: np.ndarray, lists: np.ndarray):
    """FLOPs the tiered forward is defined to execute, by tier, with real
    (ragged) block sizes: 4*|q_i|*|k_j|*d per full and low tile, three times
    that per residual tile (A1 B1 + A1 B2 + A2 B1 for S and for P V), and
    4*|q_i|*d per skipped block.  Returns (full, res, low, skip)."""
    N, d, bq, bk = cfg.N, cfg.d, cfg.block_q, cfg.block_k
    nqb, nkb = cfg.n_qb, cfg.n_kb
    qrows = np.array([min(bq, N - i * bq) for i in range(nqb)], dtype=np.float64)
    kcols = np.array([min(bk, N - j * bk) for j in range(nkb)], dtype=np.float64)
    BH = counts.shape[0]
    full_cols = np.zeros((BH, nqb))
    res_cols = np.zeros((BH, nqb))
    low_cols = np.zeros((BH, nqb))
    n_skip = counts[..., 3].astype(np.float64)
    for bh in range(BH):
        for i in range(nqb):
            nf, nr, nl = (int(x) for x in counts[bh, i, :3])
            full_cols[bh, i] = kcols[lists[bh, i, :nf]].sum()
            res_cols[bh, i] = kcols[lists[bh, i, nf:nf + nr]].sum()
            low_cols[bh, i] = kcols[lists[bh, i, nf + nr:nf + nr + nl]].sum()
    full = 4.0 * d * (full_cols * qrows[None, :]).sum()
    res = 3.0 * 4.0 * d * (res_cols * qrows[None, :]).sum()
    low = 4.0 * d * (low_cols * qrows[None, :]).sum()
    skip = 4.0 * d * (n_skip * qrows[None, :]).sum()
    return full, res, low, skip


def workload(args, name=None):
    cfg = get_config(name or args.workload)
    if args.heads:
        cfg = cfg.with_(H=args.heads)
    return cfg


def sweep(args):
    """Forward time of the 480p-shaped layer at every sparsity-sweep point
    (FP8 low tier = 20 % of kept tiles) and its speedup over the all-full
    point, one JSON line per point (not the benchmark contract line)."""
    import precision_attention_video_b200 as pav

    dev = torch.device("cuda", 0)
    base = workload(args, "sweep0")
    Q, K, V = make_qkv(base)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    O = torch.empty_like(Qd)
    dense = 4.0 * base.B * base.H * float(base.N) ** 2 * base.d
    ref_ms = None
    for pct in (0, 30, 50, 70, 90):
        cfg = workload(args, f"sweep{pct}")
        p = pav.params_for(cfg)
        ws = pav.alloc_workspace(p, dev)
        for _ in range(args.warmup):
            pav.plan(p, Qd, Kd, Vd, ws)
            pav.forward(p, Qd, Kd, Vd, ws, O)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        fwd, pln = [], []
        for _ in range(args.steps):
            ev[0].record()
            pav.plan(p, Qd, Kd, Vd, ws)
            ev[1].record()
            pav.forward(p, Qd, Kd, Vd, ws, O)
            ev[2].record()
            torch.cuda.synchronize()
            pln.append(ev[0].elapsed_time(ev[1]))
            fwd.append(ev[1].elapsed_time(ev[2]))
        st = pav.get_status(ws)
        t = pav.plan_views(p, ws)["tier_map"].cpu().numpy()
        f = statistics.median(fwd)
        if pct == 0:
            ref_ms = f
        print(json.dumps({
            "sweep_point": pct, "tau": list(cfg.tau), "status": st,
            "tier_frac": {"full": float((t == 3).mean()), "low": float((t == 1).mean()),
                          "skip": float((t == 0).mean())},
            "ms_forward": f, "ms_plan": statistics.median(pln),
            "dense_equiv_tflops_forward": dense / (f * 1e-3) / 1e12,
            "dense_equiv_tflops_layer": dense / ((f + statistics.median(pln)) * 1e-3) / 1e12,
            "forward_speedup_vs_all_full": ref_ms / f}), flush=True)
        del ws


def tier_costs(args):
    """Forward cost of each tier on the 480p shape (``--heads`` heads, 8 by
    default): thresholds chosen so that every tile but the forced diagonal
    falls in one tier, one JSON line per case with the time per kept tile
    and SM (the price router's default tier costs are these, relative to
    the bf16 tile)."""
    import precision_attention_video_b200 as pav

    dev = torch.device("cuda", 0)
    base = get_config("480p").with_(H=args.heads or 8)
    Q, K, V = make_qkv(base)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    O = torch.empty_like(Qd)
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    cases = [("full", 2, (2.0, 2.0)), ("fp8", 1, (0.0, 2.0)), ("nvfp4", 2, (0.0, 2.0)),
             ("res", 3, (0.0, 2.0, 2.0)), ("skip", 2, (0.0, 0.0))]
    for name, low, tau in cases:
        cfg = base.with_(low=low, tau=tau)
        p = pav.params_for(cfg)
        ws = pav.alloc_workspace(p, dev)
        pav.plan(p, Qd, Kd, Vd, ws)
        for _ in range(args.warmup):
            pav.forward(p, Qd, Kd, Vd, ws, O)
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            pav.forward(p, Qd, Kd, Vd, ws, O)
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        t = pav.plan_views(p, ws)["tier_map"].cpu()
        n = {k: int((t == c).sum()) for k, c in (("full", 3), ("res", 2), ("low", 1), ("skip", 0))}
        ms = statistics.median(ts)
        kept = n["full"] + n["res"] + n["low"]
        print(json.dumps({"tier_case": name, "status": pav.get_status(ws), "ms_forward": ms, "tiles": n,
                          "us_per_kept_tile_per_sm": ms * 1e3 * n_sm / kept,
                          "us_per_cta_per_sm": ms * 1e3 * n_sm / (cfg.n_qb * cfg.H)}), flush=True)
        del ws


def plan_reuse(args):
    """Plan reuse across timesteps: on a slowly changing sequence of K inputs
    (latent_gen.make_qkv_steps, correlation rho between steps), one plan
    serves K layers (tiered_attn_prep + tiered_attn_forward on the others),
    against a fresh plan on every step.  One JSON line: time per layer both
    ways and how far the last step's output moves from the fresh plan's."""
    import precision_attention_video_b200 as pav
    from latent_gen.generator import make_qkv_steps

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = workload(args)
    k = args.reuse
    seq = [tuple(x.to(dev) for x in step) for step in make_qkv_steps(cfg, k, args.rho)]
    p = pav.params_for(cfg)
    ws = pav.alloc_workspace(p, dev)
    ws_fresh = pav.alloc_workspace(p, dev)
    O = torch.empty_like(seq[0][0])
    O_fresh = torch.empty_like(O)

    def reuse_group():
        for t, (Q, K, V) in enumerate(seq):
            (pav.plan if t == 0 else pav.prep)(p, Q, K, V, ws)
            pav.forward(p, Q, K, V, ws, O)

    def fresh_group():
        for Q, K, V in seq:
            pav.plan(p, Q, K, V, ws_fresh)
            pav.forward(p, Q, K, V, ws_fresh, O_fresh)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(args.steps):
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / k)
        return statistics.median(ts)

    ms_reuse = timed(reuse_group)
    ms_fresh = timed(fresh_group)
    st = max(pav.get_status(ws), pav.get_status(ws_fresh), key=abs)
    # both workspaces and outputs now hold the last step: compare them, and
    # each with dense attention of that step (torch SDPA, measurement only)
    rel = float((O.float() - O_fresh.float()).norm() / O_fresh.float().norm())
    Ql, Kl, Vl = seq[-1]
    dense_o = torch.nn.functional.scaled_dot_product_attention(Ql, Kl, Vl).float()
    err_reuse = float((O.float() - dense_o).norm() / dense_o.norm())
    err_fresh = float((O_fresh.float() - dense_o).norm() / dense_o.norm())
    same = float((pav.plan_views(p, ws)["tier_map"] == pav.plan_views(p, ws_fresh)["tier_map"])
                 .float().mean())
    dense = 4.0 * cfg.B * cfg.H * float(cfg.N) ** 2 * cfg.d
    print(json.dumps({
        "metric": METRIC, "mode": "plan reuse across timesteps", "workload": cfg.name,
        "every": k, "rho": args.rho, "status": st,
        "ms_per_layer_reused_plan": ms_reuse, "ms_per_layer_fresh_plan": ms_fresh,
        "dense_equiv_tflops_reused": dense / (ms_reuse * 1e-3) / 1e12,
        "dense_equiv_tflops_fresh": dense / (ms_fresh * 1e-3) / 1e12,
        "speedup": ms_fresh / ms_reuse,
        "last_step": {"rel_l2_vs_fresh_plan": rel, "tier_map_agreement": same,
                      "rel_l2_vs_dense_reused_plan": err_reuse,
                      "rel_l2_vs_dense_fresh_plan": err_fresh}}), flush=True)


def run_gpu_arm(args, rank, world, local_rank):
    import precision_attention_video_b200 as pav

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = workload(args)
    Q, K, V = make_qkv(cfg)
    p = pav.params_for(cfg)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    O = torch.empty_like(Qd)
    ws = pav.alloc_workspace(p, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        pav.plan(p, Qd, Kd, Vd, ws, stream)
        pav.forward(p, Qd, Kd, Vd, ws, O, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = pav.get_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {pav.status_string(st)}")

    views = pav.plan_views(p, ws)
    counts = views["row_counts"].cpu().numpy()
    lists = views["row_lists"].cpu().numpy()
    tiers = views["tier_map"].cpu().numpy()
    full_flops, res_flops, low_flops, skip_flops = algorithmic_attn_flops(cfg, counts, lists)

    # timed region: K whole steps, events around each forward for the roofline
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for a, b, c in ev:
            a.record(stream)
            pav.plan(p, Qd, Kd, Vd, ws, stream)
            b.record(stream)
            pav.forward(p, Qd, Kd, Vd, ws, O, stream)
            c.record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    plan_ms = [a.elapsed_time(b) for a, b, _ in ev]
    fwd_ms = [b.elapsed_time(c) for _, b, c in ev]
    st = pav.get_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {pav.status_string(st)}")

    # end to end through the public C ABI from pinned host buffers
    Qh, Kh, Vh = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    Oh = torch.empty_like(Q).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    pav.layer_from_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, O, ws, stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        pav.layer_from_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, O, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    res = {
        "total_ms": total_ms, "plan_ms": plan_ms, "fwd_ms": fwd_ms, "e2e_ms": e2e_ms,
        "clocks": clk.summary(), "full_flops": full_flops, "res_flops": res_flops,
        "low_flops": low_flops,
        "skip_flops": skip_flops,
        "tier_frac": {n: float((tiers == t).mean()) for n, t in
                      (("full", 3), ("res", 2), ("low", 1), ("skip", 0))},
        "h2d": 3 * Q.numel() * Q.element_size(), "d2h": O.numel() * O.element_size(),
    }
    return cfg, res


def cpu_baseline(cfg, budget_s: float = 20.0, threads: int = 0):
    """The oracle, as it stands, on a bounded sample of the workload: whole
    heads are routed (with the workload's router) and quantised, then query
    blocks of those heads (spread over the sequence) are attended until the
    time budget is used.  The unit is dense-equivalent TFLOPS of the query
    rows attended; input generation is not timed."""
    import oracle
    from latent_gen.generator import make_head
    from oracle import quant as Qz
    from oracle import route as Rt

    cores = threads or len(os.sched_getaffinity(0))
    rows, heads, spent = 0, 0, 0.0
    nqb = cfg.n_qb
    order = [(i * 17) % nqb for i in range(nqb)]
    while spent < budget_s and heads < cfg.H:
        q, k, v = make_head(cfg, 0, heads)
        Qh, Kh, Vh = (torch.from_numpy(x).to(torch.bfloat16).double().numpy() for x in (q, k, v))
        t = time.time()
        rt = Rt.route_head(Qh, Kh, Vh, cfg.tau, cfg.block_q, cfg.block_k,
                           router=getattr(cfg, "router", 0), price=getattr(cfg, "price", 0.0),
                           low=cfg.low, kappa=getattr(cfg, "kappa", 1.0),
                           tier_cost=getattr(cfg, "tier_cost", None))
        qt = Qz.quantize_head(Qh, Kh, Vh, cfg.low, cfg.block_q, cfg.block_k)
        spent += time.time() - t
        done = 0
        while done < nqb and spent < budget_s:
            blocks = order[done:done + cores]
            t = time.time()
            oracle.tiered_attention_head(Qh, Kh, Vh, rt, qt, cfg.low, cfg.block_q, cfg.block_k,
                                         cfg.p_offset_log2, rt["scale"], False, blocks,
                                         threads=cores, key_pack=cfg.key_pack)
            spent += time.time() - t
            rows += sum(min(cfg.block_q, cfg.N - i * cfg.block_q) for i in blocks)
            done += len(blocks)
        heads += 1
    flops = 4.0 * rows * cfg.N * cfg.d
    return {"value": flops / spent / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{heads} head(s) of the workload routed and quantised in full, {rows} of "
                      f"{cfg.B * cfg.H * cfg.N} query rows attended; {spent:.1f} s of oracle time"}


def max_over_ranks(values, world):
    """Each value's maximum over the ranks: a replicated step takes as long as
    its slowest rank.  NCCL reduces on the device, gloo on the host."""
    if world <= 1:
        return [float(v) for v in values]
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(world, dense_flops, ms):
    """Dense-equivalent TFLOP/s of the whole job: each of `world` replicas
    runs the full layer in `ms` milliseconds (the max over ranks)."""
    return world * dense_flops / (ms * 1e-3) / 1e12


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller profiling cases)")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload name (latent_gen.configs); the contract line uses 480p")
    ap.add_argument("--sweep", action="store_true",
                    help="time the sparsity sweep instead (one JSON line per point)")
    ap.add_argument("--reuse", type=int, default=0,
                    help="time plan reuse instead: one plan per K timesteps of a correlated sequence")
    ap.add_argument("--rho", type=float, default=0.99,
                    help="correlation between consecutive timesteps for --reuse")
    ap.add_argument("--tier-costs", action="store_true",
                    help="time each tier alone on the 480p shape instead (one JSON line per tier)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.tier_costs:
        tier_costs(args)
        return

    if args.sweep:
        sweep(args)
        return
    if args.reuse > 0:
        plan_reuse(args)
        return
    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    local_rank = _env_int("LOCAL_RANK", 0)
    cfg = workload(args)
    from latent_gen.configs import LOW_NAMES
    title = {"480p": "480p-video-like tiered attention layer",
             "720p": "720p-long-video-like tiered attention layer"}.get(
                 cfg.name, f"{cfg.name} tiered attention layer")
    config = {"workload": title, "B": cfg.B, "H": cfg.H,
              "N": cfg.N, "d": cfg.d, "grid_txyx": list(cfg.grid),
              "tile": [cfg.block_q, cfg.block_k], "low_tier": LOW_NAMES[cfg.low],
              **({"router": "single price", "price": cfg.price} if getattr(cfg, "router", 0) == 1
                 else {"router": "entropy retention", "kappa": cfg.kappa, "tau": list(cfg.tau)}
                 if getattr(cfg, "router", 0) == 2
                 else {"router": "cumulative pooled mass", "tau": list(cfg.tau)}),
              "logit_std": cfg.logit_std,
              "l2": f"inputs larger than L2 (Q+K+V {3 * cfg.B * cfg.H * cfg.N * cfg.d * 2 / 1e9:.2f} GB per GPU)",
              "parallelism": f"replicas x{args.gpus}"}

    if args.impl == "reference":
        if rank != 0:
            return
        t = time.time()
        per = []
        for _ in range(args.steps):
            per.append(cpu_baseline(cfg, budget_s=max(5.0, 120.0 / max(1, args.steps))))
        v = statistics.median([x["value"] for x in per])
        ms = 4.0 * cfg.B * cfg.H * cfg.N ** 2 * cfg.d / (v * 1e12) * 1e3
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": UNIT, "cores": per[0]["cores"],
                                 "kind": "oracle", "sample": per[0]["sample"]},
                "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "wall_s": time.time() - t}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    cfg, r = run_gpu_arm(args, rank, world, local_rank)

    dense = 4.0 * cfg.B * cfg.H * float(cfg.N) ** 2 * cfg.d
    step_ms = r["total_ms"] / args.steps
    fwd_ms = statistics.mean(r["fwd_ms"])
    step_ms, fwd_ms, e2e_ms = max_over_ranks([step_ms, fwd_ms, r["e2e_ms"]], world)
    peaks, peak_src = load_peaks()
    p_bf16, peak_kind = bf16_peak(peaks, r["clocks"])
    # Full tiles and skip chunks run on the bf16 pipe; NVFP4 tiles (low and
    # residual) on the FP4 pipe and FP8 tiles on the FP8 pipe, whose peaks are
    # taken as 4x and 2x the measured bf16 one (the nominal ratios).
    p_fp4 = 4.0 * p_bf16
    p_low = {1: 2.0 * p_bf16, 2: p_fp4, 3: p_fp4}.get(cfg.low, p_bf16)
    executed = r["full_flops"] + r["res_flops"] + r["low_flops"] + r["skip_flops"]
    t_min = ((r["full_flops"] + r["skip_flops"]) / (p_bf16 * 1e12) + r["res_flops"] / (p_fp4 * 1e12)
             + r["low_flops"] / (p_low * 1e12))
    peak = executed / t_min / 1e12          # blended tensor peak of this launch's FLOP mix
    achieved = executed / (fwd_ms * 1e-3) / 1e12
    traffic = None
    if ATTN_TRAFFIC["source_sha1"] == attn_source_sha1() and cfg.name == WORKLOAD and cfg.H == 40:
        traffic = ATTN_TRAFFIC["bytes_per_launch"]

    if rank == 0:
        line = {
            "metric": METRIC, "value": whole_job_tflops(world, dense, step_ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config,
            "ms_plan": statistics.mean(r["plan_ms"]), "ms_forward": fwd_ms,
            "tier_frac": r["tier_frac"],
            "roofline": {"kernel": f"tiered_attn_forward ({attn_kernel_name(cfg)})", "bound": "tensor",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": (f"blend of {peak_src} bf16 {peak_kind} "
                                         f"{p_bf16:.1f}, nvfp4 = 4x and native fp8 = 2x "
                                         "that (nominal ratios), weighted by the launch's "
                                         "FLOPs per tier"),
                         "flops_per_launch": executed,
                         "flops_by_tier": {"full": r["full_flops"], "res": r["res_flops"],
                                           "low": r["low_flops"], "skip": r["skip_flops"]}},
            "e2e": {"value": whole_job_tflops(world, dense, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                    "ms_per_step": e2e_ms},
            "gpu_launches": 4 * args.steps,
            "clocks": r["clocks"],
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(cfg)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
