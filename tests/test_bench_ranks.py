"""bench.py's multi-rank host logic on CPU: two gloo ranks on 127.0.0.1 take
the slowest rank's time, count every rank's work in the whole-job rate, and
draw distinct replica seeds (no data-path collective exists: the layer has no
cross-token exchange, so ranks run independent replicas)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ms_of_rank, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        r, lr, w = bench.rank_env()
        slow = bench.max_over_ranks(dist, ms_of_rank[rank])
        rate = bench.whole_job_rate(5 * 10, w, slow)
        out[rank] = (r, lr, w, slow, rate, bench.replica_seed(1, r))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_work():
    world, port = 2, _free_port()
    ms = [2.5, 4.0]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, ms, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        r, lr, w, slow, rate, seed = res[rank]
        assert (r, lr, w) == (rank, rank, world)
        assert slow == pytest.approx(max(ms))  # every rank sees the slowest rank's time
        assert rate == pytest.approx(5 * 10 * world / (max(ms) / 1e3))
    assert res[0][5] != res[1][5]  # independent replicas draw different data


def test_single_rank_is_unchanged():
    import bench
    assert bench.max_over_ranks(None, 3.25) == 3.25
    assert bench.whole_job_rate(50, 1, 1000.0) == pytest.approx(50.0)
