"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each timing its own
independent problem (weak scaling, no collective on the data path); the whole-job value
is the units of all ranks over the max-over-ranks time."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r processed (r + 1) * 1000 units in (r + 1) * 10 ms of device time
        rate, ms_max = bench.whole_job_rate((rank + 1) * 1000.0, (rank + 1) * 10.0, world)
        bench.barrier(world)
        out[rank] = (rate, ms_max, bench.reduce_max(float(rank), world), bench.reduce_sum(1.0, world))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        rate, ms_max, mx, sm = out[rank]
        assert ms_max == pytest.approx(20.0)            # max over ranks
        assert rate == pytest.approx(3000.0 / 0.020)    # all units / max time
        assert mx == 1.0 and sm == 2.0


def test_single_rank_is_identity():
    import bench
    rate, ms = bench.whole_job_rate(500.0, 5.0, 1)
    assert ms == 5.0 and rate == pytest.approx(100000.0)
