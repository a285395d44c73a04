"""Multi-process host logic on CPU: world_size-2 gloo ranks (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from block_sparse_cross_sparvar_b200 import multi


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = multi.max_over_ranks([1.0 + rank, 10.0 - rank])
        sm = multi.sum_over_ranks([2.0 * (rank + 1)])
        tput, tmax = multi.job_throughput(1e12 * (rank + 1), 1.0 + rank)
        dist.barrier()
        q.put((rank, mx, sm, tput, tmax))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_times_and_flops():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, tput, tmax in results:
        assert mx == [2.0, 10.0]
        assert sm == [6.0]
        # 3e12 FLOP over the slowest rank's 2 ms
        assert tmax == 2.0 and abs(tput - 1500.0) < 1e-9


@pytest.mark.parametrize("B,H,world", [(2, 16, 8), (2, 16, 3), (1, 5, 4), (3, 1, 2)])
def test_shard_pairs_partition(B, H, world):
    seen = []
    for r in range(world):
        a, b = multi.shard_pairs(B, H, r, world)
        assert 0 <= a <= b <= B * H
        seen.extend(range(a, b))
    assert seen == list(range(B * H))
    sizes = [multi.shard_pairs(B, H, r, world)[1] - multi.shard_pairs(B, H, r, world)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_single_process_identity():
    assert multi.max_over_ranks([3.0]) == [3.0]
    tput, t = multi.job_throughput(2e12, 4.0)
    assert abs(tput - 500.0) < 1e-9 and t == 4.0
