"""The benchmark's N > 1 bookkeeping on CPU: world_size-2 gloo ranks (no GPU).

With tokens sharded across GPUs and weights replicated the layer has no exchange step, so
`bench.py --gpus N` runs N independent replicas; its only collectives are the timing barrier
and the max-over-ranks reduction, and rank 0 alone prints.  These tests run exactly those
pieces as two processes over gloo on 127.0.0.1.
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


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, world, "cpu")
        value = bench.job_throughput(world, 4096, 20, ms)
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_max_time_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 15.0                      # the max over ranks, identical on every rank
        assert value == pytest.approx(2 * 4096 * 20 / 0.015)  # all ranks' tokens / the slowest time


def test_single_rank_throughput_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(1, 1, 1000, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_prints_only_on_rank_zero():
    # under torchrun every rank runs bench.py; only rank 0 times the oracle and prints
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny_f32", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "1", "--warmup", "0", "--cpu-sample-tokens", "4"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
