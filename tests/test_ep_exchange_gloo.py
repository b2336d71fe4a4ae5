"""Expert parallelism's all-to-all layout and volume on CPU (no GPU).

Two or four gloo ranks each route and claim slots on their own batch with
the oracle, all-gather their kept counts, place their rows with the layout
rule (ep.layout_host, the host restatement the GPU test checks moe_ep_layout
against) and exchange the rows with torch.distributed.  Every receiver's
buffer must be tiled exactly -- expert-major, source GPU order inside an
expert, claim order inside a source -- and hold exactly the rows the
senders' dispatch kept for its experts.  The bytes that actually crossed
ranks must equal ep.a2a_bytes, and a2a_bytes must reproduce the pages'
all-to-all volume (CMU 10-423 Lecture 16, section 6.2 and exercise 4)."""
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


def _rank(rank, world, port, out, N, k, T, d):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from mixture_experts_sparse_b200 import inputs
    from mixture_experts_sparse_b200.ep import a2a_bytes, layout_host

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E = N // world
        L = inputs.make_layer(T=T, d_model=d, d_ff=16, n_experts=N, top_k=k, dtype="f32", seed=11,
                              x_seed=100 + rank, router_bias=np.linspace(0.7, 0.0, N).astype(np.float32))
        C = oracle.capacity(T, N, k, 1.0)
        r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
        dd = oracle.dispatch(r["idx"], N, C)
        kt, kr = np.nonzero(dd["drop"] == 0)
        rows = dd["offsets"][r["idx"][kt, kr]] + dd["pos"][kt, kr]
        row_token = np.empty(int(dd["offsets"][-1]), np.int64)
        row_token[rows] = kt
        kept_all = [torch.empty(N, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(kept_all, torch.from_numpy(dd["kept"].astype(np.int32)))
        kept_all = [t.numpy() for t in kept_all]
        dst, recv = layout_host(kept_all, rank)
        # messages: for every destination GPU, (destination row, token id tag, x row)
        send = [[] for _ in range(world)]
        off = dd["offsets"]
        for e in range(N):
            h = e // E
            for q in range(int(off[e]), int(off[e + 1])):
                t = int(row_token[q])
                send[h].append((dst[e] + q - int(off[e]), rank * 10 ** 6 + t, e, L["x"][t]))
        # exchange by all-gather of every rank's messages (gloo; small sizes)
        got = [None] * world
        dist.all_gather_object(got, send)
        incoming = [msg for s in range(world) for msg in got[s][rank]]
        R = recv[-1]
        buf_tag = np.full(R, -1, np.int64)
        buf_e = np.full(R, -1, np.int64)
        buf_x = np.zeros((R, d), np.float32)
        for (row, tag, e, xv) in incoming:
            assert 0 <= row < R and buf_tag[row] == -1, "overlapping or out-of-range receive row"
            buf_tag[row], buf_e[row], buf_x[row] = tag, e, xv
        crossed = sum(len(send[h]) for h in range(world) if h != rank) + \
            sum(len(got[s][rank]) for s in range(world) if s != rank)
        out[rank] = dict(recv=recv, tag=buf_tag, e=buf_e, x=buf_x, kept_all=np.stack(kept_all),
                         bytes=a2a_bytes(kept_all, rank, d, 4), crossed=crossed)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,k", [(2, 6, 1), (2, 4, 2), (4, 8, 2), (4, 4, 1)])
def test_all_to_all_layout_tiles_each_receiver(world, N, k):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from mixture_experts_sparse_b200 import inputs
    T, d = 300, 8
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out, N, k, T, d), nprocs=world, start_method="spawn", join=True)
    E = N // world
    # the expected receive buffer of every GPU, from each source's oracle dispatch
    want_tags = {h: [] for h in range(world)}
    want_x = {h: [] for h in range(world)}
    per_src = []
    for s in range(world):
        L = inputs.make_layer(T=T, d_model=d, d_ff=16, n_experts=N, top_k=k, dtype="f32", seed=11, x_seed=100 + s,
                              router_bias=np.linspace(0.7, 0.0, N).astype(np.float32))
        C = oracle.capacity(T, N, k, 1.0)
        r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
        dd = oracle.dispatch(r["idx"], N, C)
        kt, kr = np.nonzero(dd["drop"] == 0)
        rows = dd["offsets"][r["idx"][kt, kr]] + dd["pos"][kt, kr]
        row_token = np.empty(int(dd["offsets"][-1]), np.int64)
        row_token[rows] = kt
        per_src.append((dd, row_token, L["x"]))
    for h in range(world):
        for j in range(E):
            e = h * E + j
            for s in range(world):
                dd, row_token, x = per_src[s]
                for q in range(int(dd["offsets"][e]), int(dd["offsets"][e + 1])):
                    want_tags[h].append(s * 10 ** 6 + int(row_token[q]))
                    want_x[h].append(x[row_token[q]])
    for h in range(world):
        o = out[h]
        assert (o["tag"] >= 0).all(), "receive buffer has holes"
        np.testing.assert_array_equal(o["tag"], np.array(want_tags[h], np.int64))
        np.testing.assert_array_equal(o["x"], np.array(want_x[h], np.float32).reshape(-1, d))
        # expert-major: local expert j fills [recv[j], recv[j + 1])
        for j in range(E):
            assert (o["e"][o["recv"][j]:o["recv"][j + 1]] == h * E + j).all()
        assert o["crossed"] * d * 4 == o["bytes"]


def test_volume_reproduces_the_pages_figures(golden):
    import sys
    sys.path.insert(0, ROOT)
    from mixture_experts_sparse_b200.ep import a2a_bytes
    g = golden("all_to_all_volume.txt")
    T, k, d, eb = g["T_per_gpu"], g["k"], g["d"], g["elem_bytes"]
    assert T * k * d * eb / 1e6 == pytest.approx(g["dispatch_total_mb"], abs=0.5)
    for G, key in ((8, "per_gpu_mb_8"), (64, "per_gpu_mb_64")):
        N = G   # one expert per GPU; uniform routing, nothing dropped
        kept_all = [[T * k // N] * N for _ in range(G)]
        per_gpu = a2a_bytes(kept_all, 3, d, eb) / 1e6
        assert per_gpu == pytest.approx(g[key], abs=0.5), (G, per_gpu)
        if G == 8:
            assert per_gpu / 2 == pytest.approx(g["dispatch_remote_mb_8"], abs=0.5)
