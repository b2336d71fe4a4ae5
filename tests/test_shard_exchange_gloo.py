"""The sharded routing group's exchange on CPU: two or three gloo ranks each
hold a contiguous shard (uneven; one shard of a single token), all-gather
their claim counts, derive their claim base and claim slots from it (oracle
arithmetic), and together reproduce the oracle's single-group dispatch
exactly, for top-1 and top-2 (no GPU)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out, k, bounds):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from mixture_experts_sparse_b200 import inputs
    from mixture_experts_sparse_b200.shard import dist_all_gather

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, N = bounds[-1], 6
        L = inputs.make_layer(T=T, d_model=32, d_ff=16, n_experts=N, top_k=k, dtype="f32", seed=5)
        C = oracle.capacity(T, N, k, 1.0)
        a, b = bounds[rank], bounds[rank + 1]
        r = oracle.route(L["x"][a:b], L["w_r"], None, k)
        counts = np.zeros((k, N), np.int32)
        for rr in range(k):
            counts[rr] = np.bincount(r["idx"][:, rr], minlength=N)
        gather = dist_all_gather()
        all_counts = gather(torch.from_numpy(counts)).numpy()       # [S, k, N]
        base0 = all_counts[:rank, 0].sum(0)
        local = oracle.dispatch(r["idx"], N, 10 ** 9)                 # local claim numbers (no capacity)
        pos = local["pos"].copy()
        pos[:, 0] += base0[r["idx"][:, 0]]
        if k == 2:
            base1 = all_counts[:, 0].sum(0) + all_counts[:rank, 1].sum(0)
            pos[:, 1] = (pos[:, 1] - counts[0][r["idx"][:, 1]]) + base1[r["idx"][:, 1]]
        out[rank] = (a, b, pos, (pos >= C).astype(np.uint8))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("k,bounds", [(2, [0, 430, 900]), (1, [0, 300, 301, 1000]), (2, [0, 1, 600, 777])])
def test_rank_exchange_reproduces_the_group_dispatch(k, bounds):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from mixture_experts_sparse_b200 import inputs
    world, port = len(bounds) - 1, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out, k, bounds), nprocs=world, start_method="spawn", join=True)
    T, N = bounds[-1], 6
    L = inputs.make_layer(T=T, d_model=32, d_ff=16, n_experts=N, top_k=k, dtype="f32", seed=5)
    C = oracle.capacity(T, N, k, 1.0)
    full = oracle.dispatch(oracle.route(L["x"], L["w_r"], None, k)["idx"], N, C)
    pos = np.concatenate([out[r][2] for r in range(world)])
    drop = np.concatenate([out[r][3] for r in range(world)])
    np.testing.assert_array_equal(pos, full["pos"])
    np.testing.assert_array_equal(drop, full["drop"])
