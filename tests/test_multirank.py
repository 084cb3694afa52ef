"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (127.0.0.1).
The job time is the max over ranks and the whole-job rate counts every rank's
work; the default multi-GPU mode splits the heads of one chunk over the ranks
and all-gathers O in place; the other mode runs one chunk per rank."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms = [3.0 + rank, 10.0 - 4 * rank]           # rank 0: (3, 10), rank 1: (4, 6)
    got = bench.reduce_max(ms)
    value = bench.job_throughput(world, 2.0e12, got[0])
    out[rank] = (got, value, bench.rank_seed(3, rank))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_every_rank():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        got, value, seed = res[rank]
        assert got == [4.0, 10.0]
        assert value == pytest.approx(world * 2.0e12 / 4.0e-3)
        assert seed == 1003 + rank
    assert res[0][2] != res[1][2]  # the ranks run different chunks


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_throughput(1, 1e12, 1.0) == pytest.approx(1e15)


def _heads_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ok = []
    for B in (1, 2):
        H, N, d = 24, 8, 4
        full = torch.arange(B * H * N * d, dtype=torch.float32).view(B, H, N, d)
        h0, h1 = bench.head_range(H, world, rank)
        # this rank's heads are written into its slice of the gathered buffer,
        # which the all-gather then fills in place
        o_all = torch.full((world * B, h1 - h0, N, d), -1.0)
        mine = o_all[rank * B:(rank + 1) * B]
        mine.copy_(full[:, h0:h1])
        got = bench.gather_heads(o_all, mine, world)
        ok.append(bool(torch.equal(got, full)))
    out[rank] = ((h0, h1), all(ok))
    dist.barrier()
    dist.destroy_process_group()


def test_heads_split_and_gather_over_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_heads_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == ((0, 12), True) and res[1] == ((12, 24), True)


def test_head_range_rejects_uneven_splits():
    sys.path.insert(0, ROOT)
    import bench
    assert [bench.head_range(24, 8, r) for r in (0, 7)] == [(0, 3), (21, 24)]
    with pytest.raises(ValueError):
        bench.head_range(24, 5, 0)
