"""The N > 1 host path of bench.py on CPU: two gloo ranks.

With more than one GPU each rank runs its share of one problem (its own zigzag shards;
the collectives are covered by tests/test_sharded_cpu.py); what spans ranks in the
bench is the timing rule -- the job's time is the slowest rank's -- and the whole-job
value, the sum of every rank's work over that time.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 17.25][rank]
        ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        out[rank] = (ms, bench.job_tflops(1e12, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_value():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        ms, value = out[r]
        assert ms == 17.25
        assert abs(value - 2 * 1e12 / 17.25e-3 / 1e12) < 1e-9


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert abs(bench.job_tflops(2e12, 1, 2.0) - 1000.0) < 1e-9
