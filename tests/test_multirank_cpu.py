"""The benchmark's multi-process plumbing on CPU: two gloo ranks (one process
per rank, rendezvous on 127.0.0.1) reduce their step times with a max and
their token counts with a sum, exactly as bench.py does under torchrun with one
replica per GPU (the path has no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 10.0 + 5.0 * rank                 # rank 1 is the slower one
    tokens = 1000 * (rank + 1)
    t_max = bench.reduce_over_ranks(ms, torch.device("cpu"), "max")
    tok = bench.reduce_over_ranks(tokens, torch.device("cpu"), "sum")
    q.put((rank, t_max, tok))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reduction_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t_max, tok in res:
        assert t_max == 15.0          # time = max over ranks
        assert tok == 3000.0          # work = sum over ranks


def test_single_process_reduction_is_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, torch.device("cpu")) == 3.5
