"""Host logic of the multi-rank benchmark on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` runs its own replica of the workload (the
path has no exchange step); the job's time is the slowest rank's and the
throughput counts the units of every rank.  Also: the reference arm prints
only on rank 0 and the other ranks exit without work.
"""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _rank_main(rank, world, port, values, out_dir):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(values[rank], None, world)
        tput = bench.job_throughput(8, world, 10, m)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": m, "tput": tput}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_slowest_rank_sets_the_time(tmp_path):
    values = [3.25, 7.5]  # per-rank total ms
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r in res:
        assert r["max"] == pytest.approx(7.5)
        # 2 ranks x 8 sequences x 10 steps over 7.5 ms
        assert r["tput"] == pytest.approx(2 * 8 * 10 / 7.5e-3)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(4.0) == 4.0
    assert bench.job_throughput(8, 1, 5, 2.0) == pytest.approx(8 * 5 / 2e-3)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""
