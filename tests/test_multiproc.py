"""Host logic of the multi-GPU path on CPU with world-size-2 gloo process groups:
every rank owns a different batch of requests of the same shape (independent problems,
no data-path collective) and the job time is the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    case = bench.rank_case("tiny_b2_h16", rank)
    t = bench.max_over_ranks(10.0 + rank, world)              # rank 1 is slower
    digest = float(np.asarray(case.kv[:2], dtype=np.float64).sum())
    results[rank] = (t, case.batch, case.h_q, list(case.cache_seqlens), digest)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_sharding_and_max_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, results), nprocs=2, start_method="spawn", join=True)
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 11.0                             # both ranks see the slowest rank's time
    assert r0[1:4] == r1[1:4]                                 # same shapes and cache lengths
    assert r0[4] != r1[4]                                     # different request contents
