"""bench.py's multi-rank host logic on CPU: two gloo ranks in separate processes.

The layer runs as independent replicas, one per GPU, with no data-path
collective; the only cross-rank steps are the barriers around the timed region
and the max over ranks of the device times, from which rank 0 reports the
whole job's throughput.  Those steps are checked here without a GPU.
"""

import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        dist.barrier()
        # rank r "measured" step 10 + r ms, forward 5 - r ms, e2e 7 (r + 1) ms
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 7.0 * (rank + 1)], world)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "tflops": bench.whole_job_tflops(world, 4.0e12, got[0])}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_with_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        # every rank holds the slowest rank's figures
        assert r["max"] == [11.0, 5.0, 14.0]
        # two replicas of 4 TFLOP in 11 ms: 2 * 4e12 / 11e-3 / 1e12 TFLOP/s
        assert r["tflops"] == pytest.approx(2 * 4.0e12 / 11e-3 / 1e12, rel=1e-12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3, 2.5], 1) == [3.0, 2.5]
    assert bench.whole_job_tflops(1, 2.0e12, 4.0) == pytest.approx(500.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
