"""The N > 1 path of bench.py on CPU: world_size 2 gloo ranks (127.0.0.1), each a replica with its
own timing; the job's time is the max over ranks and its throughput the sum of the replicas'
units over that time.  No collective is on the data path (replicas only)."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms = [4.5, 7.25][rank]                     # this replica's device time
    job_ms = bench.max_over_ranks(ms, world)
    rate = bench.replica_rate(1000, world, job_ms / 1000.0)
    out[rank] = (job_ms, rate)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_replicas_take_the_max_time():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        job_ms, rate = res[r]
        assert job_ms == 7.25
        assert abs(rate - 2 * 1000 / 7.25e-3) < 1e-6


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_rate(100, 1, 0.5) == 200.0
