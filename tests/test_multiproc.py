"""The multi-GPU path of bench.py is independent replicas: the only exchange
is the max-over-ranks time and the summed work.  Exercised here with two gloo
ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from paged_kv_cache_438_b200 import inputs as I
        ms, kv, ss = bench.aggregate_ranks(10.0 + rank, 1000 * (rank + 1), 64, world, torch.device("cpu"))
        spec = I.WORKLOADS["llama3_8b"]
        ctx = I.context_lens(spec, I.generator(spec["seed"] + bench.replica_seed_offset(rank)))
        results[rank] = (ms, kv, ss, ctx.tolist())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_as_replicas():
    world = 2
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        r = dict(results)
    for rank in range(world):
        ms, kv, ss, _ = r[rank]
        assert ms == 11.0                 # slowest rank
        assert kv == 1000 + 2000          # bytes of both replicas
        assert ss == 128                  # sequence-steps of both replicas
    assert r[0][3] != r[1][3]             # each rank decodes its own batch


def test_single_rank_passthrough():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_ranks(3.0, 5, 7, 1, None) == (3.0, 5.0, 7.0)
