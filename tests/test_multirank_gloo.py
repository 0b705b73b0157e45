"""Host-side logic of the N>1 bench path on CPU: two gloo ranks.

The work splits into independent (batch, KV-group) units with no data-path
collective; the only exchange is the max-over-ranks reduction of timings."""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_env()
        units = bench.shard_units(16, r, w)
        gathered = [None] * world
        dist.all_gather_object(gathered, units)
        mx = bench.reduce_max(10.0 + rank)   # per-rank "time"
        bench.barrier()
        q.put((rank, w, sorted(sum(gathered, [])), mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_max_reduction():
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
    for rank, world, all_units, mx in res:
        assert world == 2
        assert all_units == list(range(16))      # every unit exactly once across ranks
        assert mx == 11.0                          # max over ranks


def test_attended_flop_count_matches_closed_form():
    import bench
    from gated_block_sparse_flashattention_b200 import workloads
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    fwd, bwd = bench.attended_flops(w)
    assert abs(fwd / 1e9 - 125.2) < 0.1 and abs((fwd + bwd) / 1e9 - 438.1) < 0.2
