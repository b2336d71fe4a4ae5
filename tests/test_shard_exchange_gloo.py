"""The sharded routing group's exchange on CPU: two gloo ranks each hold a
contiguous shard, all-gather their claim counts, derive their claim base and
claim slots from it (oracle arithmetic), and together reproduce the oracle's
single-group dispatch exactly (no GPU)."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
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
        T, N, k = 900, 6, 2
        L = inputs.make_layer(T=T, d_model=32, d_ff=16, n_experts=N, top_k=k, dtype="f32", seed=5)
        C = oracle.capacity(T, N, k, 1.0)
        bounds = [0, 430, T]
        a, b = bounds[rank], bounds[rank + 1]
        r = oracle.route(L["x"][a:b], L["w_r"], None, k)
        counts = np.zeros((k, N), np.int32)
        for rr in range(k):
            counts[rr] = np.bincount(r["idx"][:, rr], minlength=N)
        gather = dist_all_gather()
        all_counts = gather(torch.from_numpy(counts)).numpy()       # [S, k, N]
        base0 = all_counts[:rank, 0].sum(0)
        base1 = all_counts[:, 0].sum(0) + all_counts[:rank, 1].sum(0)
        local = oracle.dispatch(r["idx"], N, 10 ** 9)                 # local claim numbers (no capacity)
        pos = local["pos"].copy()
        pos[:, 0] += base0[r["idx"][:, 0]]
        pos[:, 1] = (pos[:, 1] - counts[0][r["idx"][:, 1]]) + base1[r["idx"][:, 1]]
        out[rank] = (a, b, pos, (pos >= C).astype(np.uint8))
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_reproduces_the_group_dispatch():
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from mixture_experts_sparse_b200 import inputs
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    T, N, k = 900, 6, 2
    L = inputs.make_layer(T=T, d_model=32, d_ff=16, n_experts=N, top_k=k, dtype="f32", seed=5)
    C = oracle.capacity(T, N, k, 1.0)
    full = oracle.dispatch(oracle.route(L["x"], L["w_r"], None, k)["idx"], N, C)
    pos = np.concatenate([out[0][2], out[1][2]])
    drop = np.concatenate([out[0][3], out[1][3]])
    np.testing.assert_array_equal(pos, full["pos"])
    np.testing.assert_array_equal(drop, full["drop"])
