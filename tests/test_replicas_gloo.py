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


def _heads_rank(rank, world, port, out):
    """One rank of a head-sharded generation: its share of the PCSP score,
    the benchmark's all-reduce, then the split."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import numpy as np
    import bench
    import oracle
    H, N, L, k = 8, 96, 16, 29
    g = torch.Generator()
    g.manual_seed(7)
    P = torch.rand(H, N, L, generator=g)       # the same probabilities on every rank
    content = torch.zeros(L, dtype=torch.uint8)
    content[1:L - 1] = 1
    h0, h1 = bench.head_range(H, world, rank)
    score = torch.from_numpy(np.ascontiguousarray(oracle.partition_accumulate(P[h0:h1], content)))
    bench.score_all_reduce(score)
    full = oracle.partition_accumulate(P, content)
    err = float(np.abs(score.numpy() - full).max() / np.abs(full).max())
    idx_rank = oracle.partition_select(score.numpy(), k)[0].tolist()
    idx_full = oracle.partition_select(full, k)[0].tolist()
    dist.barrier()
    out[rank] = (err, idx_rank, idx_full, (h0, h1))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_head_sharded_split_matches_one_process():
    """Head sharding of one generation: each rank sums the score over its own
    heads, one all-reduce completes it, and every rank then makes the same
    S/C split as a single process over all heads."""
    import bench
    assert [bench.head_range(24, 8, r) for r in (0, 7)] == [(0, 3), (21, 24)]
    with pytest.raises(ValueError):
        bench.head_range(24, 16, 0)
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_heads_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0][3] == (0, 4) and res[1][3] == (4, 8)
    for r in range(world):
        err, idx_rank, idx_full, _ = res[r]
        assert err <= 1e-14
        assert idx_rank == idx_full
    assert res[0][1] == res[1][1]


def _cfg_rank(rank, world, port, out):
    """One rank of a generation split by guidance branch: rank 0 (cond)
    makes the split from its scores, the benchmark's broadcast hands it to
    rank 1 (uncond); the two branch predictions are then gathered on both
    ranks for the guidance combine."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import types
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import numpy as np
    import bench
    import oracle
    H, N, L, k, F = 4, 96, 16, 29, 8
    g = torch.Generator()
    g.manual_seed(11)
    P = torch.rand(H, N, L, generator=g)
    eps = [torch.randn(N, F, generator=g), torch.randn(N, F, generator=g)]  # cond, uncond
    content = torch.zeros(L, dtype=torch.uint8)
    content[1:L - 1] = 1
    tr = types.SimpleNamespace(idx_s=torch.zeros(k, dtype=torch.int32), idx_c=torch.zeros(N - k, dtype=torch.int32),
                               s=torch.zeros(N), eps_c=torch.zeros(N, F), eps_u=torch.zeros(N, F),
                               eps_own=eps[rank].clone())
    if rank == 0:  # only the cond branch has a prompt to score the tokens against
        s_idx, c_idx, sv = oracle.partition_select(oracle.partition_accumulate(P, content), k)
        tr.idx_s.copy_(torch.from_numpy(s_idx))
        tr.idx_c.copy_(torch.from_numpy(c_idx))
        tr.s.copy_(torch.from_numpy(sv))
    bench.split_broadcast(tr)
    bench.eps_all_gather(tr)
    cfg = oracle.sw_cfg(tr.eps_c.double(), tr.eps_u.double(), tr.s, 3.0, 5.0)
    ref_split = oracle.partition_select(oracle.partition_accumulate(P, content), k)
    ref_cfg = oracle.sw_cfg(eps[0].double(), eps[1].double(), torch.from_numpy(ref_split[2]), 3.0, 5.0)
    dist.barrier()
    out[rank] = (tr.idx_s.tolist() == ref_split[0].tolist() and tr.idx_c.tolist() == ref_split[1].tolist()
                 and bool(np.array_equal(tr.s.numpy(), ref_split[2])),
                 bool(torch.equal(tr.eps_c, eps[0]) and torch.equal(tr.eps_u, eps[1])),
                 bool(np.array_equal(cfg, ref_cfg)))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_guidance_branch_split():
    """Guidance-branch sharding of one generation: the uncond rank receives
    the cond rank's split and sensitivity score exactly, both ranks end up
    with both branch predictions, and their guidance combine equals the
    single-process one."""
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_cfg_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for r in range(world):
        assert res[r] == (True, True, True), (r, res[r])
