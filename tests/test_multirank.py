"""The multi-rank path of bench.py on CPU (gloo, world size 2): every rank
takes the same collective steps, timings reduce to the slowest rank, the job
value counts all ranks' work over that time, and each rank quantizes its own
seeded activations.  The GPU path shards by tokens with no data-path
collective, so this host logic is all that N > 1 adds."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench._dist()
        assert (w, r, local) == (world, rank, rank)
        bench._barrier(w)
        ms = 1.5 + rank  # rank 1 is the slow one
        ms_max = bench._max_over_ranks(w, ms, torch.device("cpu"))
        wl = workloads.WORKLOADS["pr1"]
        x = bench.rank_x_operand(wl, rank).make()
        digest = float(x.float().abs().sum())
        q.put((rank, ms_max, bench.job_tflops(w, 2e12, ms_max), digest))
        bench._barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_ranks_on_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    (_, m0, v0, d0), (_, m1, v1, d1) = res
    assert m0 == m1 == 2.5  # max over ranks
    assert v0 == v1 == pytest.approx(2 * 2e12 / 2.5e-3 / 1e12)
    assert d0 != d1  # each rank has its own activations
