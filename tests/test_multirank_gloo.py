"""Host-side logic of the N>1 bench path on CPU: two gloo ranks.

Every rank runs a replica of the step on its own batch (seeded by the rank),
with no data-path collective; the only exchange is the max-over-ranks
reduction of the timed region, from which the whole-job throughput follows."""

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
    from gated_block_sparse_flashattention_b200 import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w_, r, lr = bench.dist_env()
        # Each rank builds its own batch of the step (seeded by its rank), as the bench's replicas do.
        wl = workloads.custom("gloo", "bf16", B=1, Hq=4, Hkv=1, d=128, T=128, K=2)
        inp = bench.rank_inputs(wl, r)
        fp = float(inp["Q"].float().sum()) + float(inp["s"].sum())
        prints = [None] * world
        dist.all_gather_object(prints, fp)
        mx = bench.reduce_max(10.0 + rank)   # per-rank timed region (ms)
        value = bench.job_throughput(1e12, 4, mx, w_)
        bench.barrier()
        q.put((rank, w_, lr, prints, mx, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_reduction():
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
    from gated_block_sparse_flashattention_b200 import workloads
    wl = workloads.custom("gloo", "bf16", B=1, Hq=4, Hkv=1, d=128, T=128, K=2)
    expect = []
    for seed in range(2):
        inp = workloads.make_training_inputs(wl, seed=seed)
        expect.append(float(inp["Q"].float().sum()) + float(inp["s"].sum()))
    assert expect[0] != expect[1]
    for rank, world, local, prints, mx, value in res:
        assert world == 2 and local == rank
        assert prints == expect                    # rank r works on the batch seeded with r
        assert mx == 11.0                          # the slowest rank's timed region
        assert abs(value - 2 * 1e12 * 4 / 11e-3 / 1e12) < 1e-9   # every rank's steps over that time


def test_attended_flop_count_matches_closed_form():
    import bench
    from gated_block_sparse_flashattention_b200 import workloads
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    fwd, bwd = bench.attended_flops(w)
    assert abs(fwd / 1e9 - 125.2) < 0.1 and abs((fwd + bwd) / 1e9 - 438.1) < 0.2
