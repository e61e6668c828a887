"""The multi-rank bench path on CPU: world_size-2 `gloo` ranks (the path does not shard,
so N GPUs run N replicas; the job's time is the slowest rank's and its throughput counts
every rank's tokens)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports step times that differ by rank; every rank must see the maxima
        mine = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        got = bench.max_over_ranks(mine, world, "cpu")
        out[rank] = (got, bench.job_throughput(world, 10, 4, got[0]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_every_replica():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        got, tput = res[rank]
        assert got == [2.0, 5.0, 0.5]              # element-wise max over ranks
        assert tput == pytest.approx(2 * 10 * 4 / 2.0)  # both replicas' tokens / slowest time


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 1.5], 1) == [3.0, 1.5]
    assert bench.job_throughput(1, 256, 1, 2.0) == 128.0
