"""The benchmark's multi-GPU mode runs independent replicas (the path has no
exchange step): each rank draws its own inputs, and the timing is the maximum
over ranks.  This checks that plumbing with two gloo ranks on the CPU."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from exact_attention_blackwell_fa_b200.inputs import Shape, make_inputs

    # replicas draw different data (seed = rank), with identical shapes
    q, _, _ = make_inputs(Shape(1, 8, 8, 2, 2, 128), seed=rank)
    local_ms = 10.0 + 5.0 * rank
    worst = bench.max_over_ranks(local_ms, device=torch.device("cpu"))
    sums = torch.tensor([float(q.float().sum())])
    gathered = [torch.zeros(1) for _ in range(world)]
    dist.all_gather(gathered, sums)
    out[rank] = (worst, [float(g) for g in gathered])
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_max_over_ranks():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()  # no fork of a process that may hold CUDA state
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    s0, s1 = out[0][1]
    assert s0 != s1  # different seeds per rank
