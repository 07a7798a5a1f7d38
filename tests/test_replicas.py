"""The replica path of bench.py (--gpus N) on CPU: world_size 2 with the gloo
backend.  Every rank runs the whole workload; the step time is the max over
ranks and the whole-job throughput sums the ranks' tokens.  No collective
touches the data path."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = [0.75, 1.25][rank]
        ms = bench.max_over_ranks(ms_local, world, torch.device("cpu"))
        tokens, value = bench.replica_throughput(32768, world, ms)
        dist.barrier()
        out[rank] = (ms, tokens, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_take_the_slowest_step_and_sum_tokens():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        ms, tokens, value = out[r]
        assert ms == pytest.approx(1.25)                 # both ranks see the slowest replica
        assert tokens == 2 * 32768
        assert value == pytest.approx(2 * 32768 / 1.25e-3)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(0.5, 1, None) == 0.5
    assert bench.replica_throughput(100, 1, 2.0) == (100, 100 / 2e-3)
