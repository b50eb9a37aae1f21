"""Multi-process plumbing of bench.py on CPU: two gloo ranks (no GPU).

Each rank gets its own batch (distinct seeded inputs), the job time is the slowest rank's, and the
whole-job rate counts every rank's work over that time.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import seeded_inputs as si
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, dist, device="cpu")
        seed = bench.rank_seed(2, rank)
        q = si.batch_item(seed, si.Q_ID, 0, (4, 2, 8), "bf16")
        digest = int(np.frombuffer(q.tobytes(), dtype=np.uint16).astype(np.int64).sum())
        rate = bench.whole_job_rate(1e9, ms_max, world)
        out.put((rank, ms_max, digest, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, d0, rate0), (r1, ms1, d1, rate1) = res
    assert ms0 == ms1 == 15.0          # max over ranks, seen identically by both
    assert d0 != d1                    # each rank has its own batch
    assert rate0 == rate1 == pytest.approx(2 * 1e9 / 0.015)


def test_single_process_defaults():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.rank_seed(5, 0) == 5
    assert bench.whole_job_rate(10.0, 1000.0, 1) == pytest.approx(10.0)
