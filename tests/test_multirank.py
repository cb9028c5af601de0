"""Host logic of the multi-GPU path on CPU: two gloo ranks, weak scaling, max over ranks.

The layer is token-parallel ("replicas only"): each rank runs its own replica on its own batch
and the job's time is the slowest rank's, so the aggregate is world * work / max(time)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, dist, "cpu")
        out[rank] = (m, bench.aggregate(2.0e12, 4, world, m))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_aggregate():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 2 ranks x 4 steps x 2 TFLOP in 15 ms
    assert res[0][1] == pytest.approx(2 * 4 * 2.0 / 15e-3)


def test_single_rank_aggregate_is_plain_rate():
    import bench

    assert bench.max_over_ranks(7.0, None, "cpu") == 7.0
    assert bench.aggregate(1.0e12, 10, 1, 10.0) == pytest.approx(1000.0)
