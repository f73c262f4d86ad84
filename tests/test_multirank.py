"""The N>1 path of bench.py on CPU: two gloo ranks combine their timings the
way the GPU ranks do (max of every time, sum of the work), each rank draws
its own inputs, and nothing else is exchanged."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from image_dits_b200.workload import WORKLOADS, make_qkv
    res = bench.combine_over_ranks(10.0 + rank, 5.0 + 2 * rank, 20.0 - rank, 1e12 * (rank + 1), dist, "cpu")
    q, _, _ = make_qkv(WORKLOADS["tiny"], "cpu", seed=bench.rank_seed(rank))
    digest = torch.tensor([float(q.float().sum())])
    all_d = [torch.zeros(1) for _ in range(world)]
    dist.all_gather(all_d, digest)
    out[rank] = (res, [float(x) for x in all_d])
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_combination():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:     # no fork of this (threaded) process
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for r in range(world):
        c, digests = res[r]
        assert c["ms_step"] == 11.0 and c["attn_ms"] == 7.0 and c["e2e_ms"] == 20.0
        assert c["flops"] == 3e12
        assert digests[0] != digests[1]          # independent batch elements


def _split_worker(rank, world, port, out):
    """One rank of a head-split call: the oracle path (permutation, mask,
    attention, inverse permutation) on this rank's heads of the call's inputs."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    from image_dits_b200.shard import head_range
    from split_case import SPLIT_WL, oracle_call
    h0, h1 = head_range(SPLIT_WL.heads, world, rank)
    o = oracle_call(SPLIT_WL, h0, h1)                       # float64 [B, h1 - h0, N, d]
    # gather the ranks' head ranges and outputs (the test's own check, not part of the path)
    ranges = [None] * world
    dist.all_gather_object(ranges, (h0, h1))
    outs = [None] * world
    dist.all_gather_object(outs, o)
    if rank == 0:
        out["ranges"] = ranges
        out["o"] = np.concatenate(outs, axis=1)
    dist.barrier()
    dist.destroy_process_group()


def test_head_split_reassembles_one_call():
    """The heads of one call divided over two gloo ranks (5 heads: 2 + 3):
    the ranges cover every head exactly once, and the ranks' oracle outputs,
    concatenated along the head axis, are bit for bit the one-process oracle
    output of the whole call."""
    import numpy as np
    from split_case import SPLIT_WL, oracle_call
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:     # no fork of this (threaded) process
        out = m.dict()
        mp.start_processes(_split_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    covered = [h for (h0, h1) in res["ranges"] for h in range(h0, h1)]
    assert covered == list(range(SPLIT_WL.heads))
    whole = oracle_call(SPLIT_WL, 0, SPLIT_WL.heads)
    assert res["o"].dtype == whole.dtype and np.array_equal(res["o"], whole)


@pytest.mark.parametrize("heads,world", [(40, 1), (40, 2), (40, 3), (40, 8), (5, 5), (7, 4)])
def test_head_range_partition(heads, world):
    from image_dits_b200.shard import head_range
    rs = [head_range(heads, world, r) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == heads
    assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
    sizes = [h1 - h0 for h0, h1 in rs]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_head_range_refuses_more_ranks_than_heads():
    from image_dits_b200.shard import head_range
    with pytest.raises(ValueError):
        head_range(2, 3, 0)
