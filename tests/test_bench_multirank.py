"""The multi-rank bench logic on CPU: two gloo ranks agree on the slowest
rank's time and on the whole-job throughput (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(local_ms[rank], world, device="cpu")
        out[rank] = (m, bench.job_tokens_per_s(1000, world, 10, m))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    local_ms = [12.5, 20.0]
    mp.start_processes(_rank, args=(world, port, local_ms, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 20.0
    # 1000 tokens x 2 ranks x 10 steps in 20 ms
    assert out[0][1] == out[1][1] == pytest.approx(1000 * 2 * 10 / 0.020)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.job_tokens_per_s(65536, 1, 200, 140.0) == pytest.approx(65536 * 200 / 0.140)
