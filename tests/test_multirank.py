"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The attention path shards by (b, h) with no exchange, so the only cross-rank steps are the
barrier and the max-over-ranks of the timings. These run here on CPU ranks; no GPU is used.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # every rank reports a different time; all must agree on the maximum
        t = bench.reduce_max(10.0 + 5.0 * rank, True, "cpu")
        lo, hi = bench.shard_heads(64, world, rank)
        dist.barrier()
        q.put((rank, t, lo, hi))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_sharding_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]
    shards = [(o[2], o[3]) for o in out]
    assert shards == [(0, 32), (32, 64)]


@pytest.mark.parametrize("BH,world", [(64, 8), (7, 3), (1, 2), (16, 16)])
def test_shards_partition_every_head_once(BH, world):
    seen = []
    for r in range(world):
        lo, hi = bench.shard_heads(BH, world, r)
        assert 0 <= lo <= hi <= BH
        seen.extend(range(lo, hi))
    assert seen == list(range(BH))


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max(3.5, False) == 3.5


def test_flop_convention():
    # fwd = 4 B H N^2 d, halved for causal, scaled by block density
    assert bench.fwd_flops(2, 3, 128, 64) == 4.0 * 2 * 3 * 128 * 128 * 64
    assert bench.fwd_flops(2, 3, 128, 64, causal=True) == 2.0 * 2 * 3 * 128 * 128 * 64
    assert bench.fwd_flops(1, 1, 256, 64, density=0.25) == 4.0 * 256 * 256 * 64 * 0.25
    wl = bench.workload(2048, 128, False, False)
    assert (wl["B"], wl["H"], wl["N"], wl["d"]) == (8, 16, 2048, 128)
