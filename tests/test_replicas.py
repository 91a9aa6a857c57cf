"""The multi-GPU path of the benchmark is replicas only (the prefill loop step has no
cross-GPU exchange): each rank runs the whole workload, the job's time is the slowest
rank's and its throughput the sum of all ranks' tokens over that time. The host logic
is checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    # rank r took (r + 1) seconds for 1000 * (r + 1) tokens
    value, t_max, units = bench.aggregate(float(rank + 1), 1000.0 * (rank + 1), dist)
    q.put((rank, value, t_max, units))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation_is_max_time_sum_units():
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
    for rank, value, t_max, units in res:
        assert t_max == 2.0 and units == 3000.0
        assert value == pytest.approx(1500.0)


def test_single_rank_aggregation():
    import bench
    assert bench.aggregate(2.0, 10.0) == (5.0, 2.0, 10.0)
