"""The N > 1 benchmark path on CPU: world_size-2 gloo ranks, each with its
own replica; the timing reduction takes the max over ranks and the whole-job
value is the sum of the ranks' work over that max time."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import bench
    from spatially_adaptive_dit_b200 import workloads as wl
    ws, r, local = bench._dist()
    assert (ws, r, local) == (world, rank, rank)
    # rank-dependent "timings": the reduction must return the max on every rank
    got = bench.max_over_ranks([10.0 + rank, 3.0 - rank], "cpu")
    # replicas draw independent inputs (the bench seeds step 1000 * rank)
    q = wl.normal((4, 8), wl.TINY, wl.OFF_Q + wl.STEP_STRIDE * 1000 * rank)
    qs = [torch.zeros_like(q, dtype=torch.float32) for _ in range(world)]
    dist.all_gather(qs, q.float())
    dist.barrier()
    out[rank] = (got, bool(not torch.equal(qs[0], qs[1])))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_reduce_max_and_independent_replicas():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for r in range(world):
        got, distinct = res[r]
        assert got == [11.0, 3.0]
        assert distinct
    import bench
    # 2 replicas of 1 TFLOP each in a slowest-rank time of 1 s -> 2 TFLOP/s
    assert abs(bench.whole_job_tflops(1e12, 2, 1000.0) - 2.0) < 1e-12
