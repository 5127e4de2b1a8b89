"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world size 2).

The decode path does not shard across GPUs (independent replicas, weak
scaling), so the only cross-rank steps are the barrier and the max-over-ranks
reduction of the timed region; these tests run them on two CPU processes.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_q) -> None:
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 1.0 + 3.0 * rank            # rank 1 is the slow one
        dist.barrier()
        t = bench.max_over_ranks(local_ms, torch.device("cpu"))
        kv = 1_000_000
        value = bench.whole_job_gbs(world, kv, t / 1e3)
        out_q.put((rank, t, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    # both ranks see the slowest rank's time, and the same whole-job value
    assert [r[1] for r in res] == [4.0, 4.0]
    assert res[0][2] == res[1][2] == pytest.approx(2 * 1_000_000 / 4e-3 / 1e9)


def test_max_over_ranks_without_process_group_is_identity():
    import torch

    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu")) == 2.5


def test_rank_inputs_weak_scaling():
    import bench
    import mla_workloads as W

    w = W.WORKLOADS["tiny"]
    a, b = bench.rank_inputs(w, 0), bench.rank_inputs(w, 1)
    for k in ("q", "kvcache", "block_table", "cache_seqlens"):
        assert a[k].shape == b[k].shape
    assert not np.array_equal(a["q"], b["q"])          # each rank its own batch
    assert a["batch"] == b["batch"] and a["h_q"] == b["h_q"]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
