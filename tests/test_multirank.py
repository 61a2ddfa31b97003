"""Multi-rank host logic of bench.py on CPU with gloo, world size 2: each rank
gets its own batch of the same shape (weak scaling), timing is the maximum
over ranks, the throughput is all ranks' units over that time, and the
reference arm does no work on ranks other than 0."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from global_attention_moe_b200 import workloads as W
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload("tiny", rank)
        x = W.make_inputs(w)
        fake_ms = 10.0 * (rank + 1)  # rank 1 is the slowest
        ms = bench.max_over_ranks(fake_ms)
        rate = bench.aggregate_rate(world, w.total_tokens, 5, ms)
        out_q.put((rank, w.seed, w.total_tokens, x.q[:4, 0, :4].copy(), ms, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, t0, q0, ms0, rate0), (r1, s1, t1, q1, ms1, rate1) = res
    assert (s0, s1) == (0, 1)                      # distinct batches
    assert t0 == t1                                # same shape on every rank
    assert not np.array_equal(q0, q1)
    assert ms0 == ms1 == 20.0                      # max over ranks
    assert rate0 == rate1 == 2 * t0 * 5 / 0.020    # all ranks' tokens / slowest time


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
