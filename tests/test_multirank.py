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
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for r in range(world):
        c, digests = res[r]
        assert c["ms_step"] == 11.0 and c["attn_ms"] == 7.0 and c["e2e_ms"] == 20.0
        assert c["flops"] == 3e12
        assert digests[0] != digests[1]          # independent batch elements
