"""Expert parallelism (moe_ep_layout, moe_ep_dispatch, moe_ep_expert_ffn)
through the C ABI.  Needs a B200.

The G GPUs of an expert-parallel layer are run one after another on one
device (ep.LocalComm: every GPU's phase completes before the next phase
starts, so no kernel waits on another): each emulated GPU routes its own
batch, the kept counts are gathered, every GPU stores its rows into the
owners' receive buffers, every owner runs only its own experts and stores the
results back.  Each GPU's output, routing and aux loss must be bit-identical
to the one-GPU forward (moe_forward) of its batch with all N experts, and
close to the oracle within the layer tolerances.  moe_ep_layout must equal
the host restatement of the layout rule.  A second test runs two processes
on the one device that exchange their receive buffers through CUDA IPC
(host-side barriers between phases), the path one process per GPU takes."""
import os
import socket

import numpy as np
import pytest

import oracle
from gpu_helpers import assert_close_out, widen_out
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.ep import EpRank, LocalComm, ep_forward, layout_host, link_local
from mixture_experts_sparse_b200.layer import MoeLayer, to_device, to_host_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    # G, T, d, d_ff, N, k, cf, act, dtype, biases
    (4, 3000, 256, 512, 8, 1, 1.25, "relu", "bf16", False),
    (2, 2000, 128, 384, 8, 2, 1.0, "swiglu", "bf16", False),
    (4, 1500, 128, 256, 4, 2, 1.25, "relu", "bf16", True),     # one expert per GPU
    (2, 700, 96, 160, 4, 1, 1.0, "relu", "f32", True),
    (2, 600, 64, 128, 6, 2, 1.5, "swiglu", "f32", False),
    (2, 32768, 512, 1024, 16, 1, 1.25, "relu", "bf16", False),  # several tiles per CTA pair on the owners
    (8, 4096, 256, 512, 8, 2, 1.25, "swiglu", "bf16", False),   # 8 GPUs, one expert each, top-2
]


def _weights(case):
    G, T, d, dff, N, k, cf, act, dtype, biases = case
    return inputs.make_layer(T=0, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, biases=biases,
                             seed=77 + N)


def _batch(case, g, Wt):
    G, T, d, dff, N, k, cf, act, dtype, biases = case
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, biases=biases,
                          seed=77 + N, x_seed=1000 * G + g)
    for key in ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2"):
        a, b = L[key], Wt[key]
        assert (a is None and b is None) or np.array_equal(a, b)
    return L


def _local(Wd, g, E):
    return {key: (None if Wd[key] is None else Wd[key][g * E:(g + 1) * E].contiguous())
            for key in ("w1", "b1", "w3", "b3", "w2", "b2")}


@pytest.mark.parametrize("case", CASES, ids=lambda c: "G{}_T{}_N{}_k{}_{}_{}".format(c[0], c[1], c[4], c[5], c[7], c[8]))
def test_ep_emulated_equals_one_gpu_forward(case):
    G, T, d, dff, N, k, cf, act, dtype, biases = case
    E = N // G
    C = nat.moe_capacity(T, N, k, cf)
    Wt = _weights(case)
    Wd = {key: to_device(Wt[key]) for key in ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")}
    Ls = [_batch(case, g, Wt) for g in range(G)]
    xs = [to_device(L["x"]) for L in Ls]
    ranks = [EpRank(G, g, T, d, dff, N, k, C, dtype, act, Wd["w_r"], Wd["b_r"], _local(Wd, g, E)) for g in range(G)]
    link_local(ranks)
    outs = ep_forward(ranks, xs, LocalComm())
    torch.cuda.synchronize()
    for r in ranks:
        nat.check(nat.moe_read_device_status(r.ws))
        nat.check(nat.moe_read_device_status(r.ws_ep))
    kept_all = [r.kept.cpu().numpy() for r in ranks]
    for g in range(G):
        dst, recv = layout_host(kept_all, g)
        np.testing.assert_array_equal(ranks[g].dst_start.cpu().numpy(), dst)
        np.testing.assert_array_equal(ranks[g].recv_offsets.cpu().numpy(), recv)
    for g in range(G):
        one = MoeLayer(T, d, dff, N, k, C, dtype, act, Ls[g])
        nat.check(one.forward(xs[g]))
        torch.cuda.synchronize()
        nat.check(nat.moe_read_device_status(one.ws))
        r = ranks[g]
        for name in ("idx", "gate", "pos", "drop", "counts", "kept", "offsets", "f", "P", "aux"):
            np.testing.assert_array_equal(getattr(r, name).cpu().numpy(), getattr(one, name).cpu().numpy(),
                                          err_msg=f"GPU {g}: {name}")
        np.testing.assert_array_equal(to_host_bits(outs[g]), to_host_bits(one.out), err_msg=f"GPU {g}: out")
    # and against the oracle, for one GPU's batch
    if T <= 4096:
        Lg = Ls[-1]
        res = oracle.forward(Lg["x"], Lg["w_r"], Lg["b_r"], {key: Lg[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")},
                             k=k, C=C, act=oracle.SWIGLU if act == "swiglu" else oracle.RELU,
                             out_dtype=oracle.BF16 if dtype == "bf16" else oracle.F32)
        got = widen_out(outs[-1]) if dtype == "bf16" else outs[-1].cpu().numpy().astype(np.float64)
        assert_close_out(got, res["out_exact"], dtype)


def test_ep_rejects_uneven_expert_split():
    cfg = nat.config(100, 64, 64, 6, 1, 20)
    assert nat.moe_ep_recv_rows(cfg, 4) == -1
    assert nat.moe_ep_workspace_bytes(cfg, 4) == 0
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    assert nat.moe_ep_layout(4, 0, 6, t, t, t) == nat.MOE_ERR_UNSUPPORTED
    assert nat.moe_ep_layout(2, 2, 6, t, t, t) == nat.MOE_ERR_INVALID_ARG


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_rank(rank, world, port, case, out):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist

    from mixture_experts_sparse_b200 import native as nat
    from mixture_experts_sparse_b200.ep import DistComm, EpRank, ep_forward, link_ipc
    from mixture_experts_sparse_b200.layer import MoeLayer, to_device, to_host_bits
    from test_gpu_ep import _batch, _local, _weights

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        G, T, d, dff, N, k, cf, act, dtype, biases = case
        E = N // G
        C = nat.moe_capacity(T, N, k, cf)
        Wt = _weights(case)
        Wd = {key: to_device(Wt[key]) for key in ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")}
        L = _batch(case, rank, Wt)
        x = to_device(L["x"])
        r = EpRank(G, rank, T, d, dff, N, k, C, dtype, act, Wd["w_r"], Wd["b_r"], _local(Wd, rank, E))
        link_ipc(r)
        comm = DistComm()
        for _ in range(2):   # twice: the second forward reuses every buffer
            ep_forward([r], [x], comm)
            torch.cuda.synchronize()
            dist.barrier()
        nat.check(nat.moe_read_device_status(r.ws_ep))
        one = MoeLayer(T, d, dff, N, k, C, dtype, act, L)
        nat.check(one.forward(x))
        torch.cuda.synchronize()
        out[rank] = bool(np.array_equal(to_host_bits(r.out), to_host_bits(one.out)))
        dist.barrier()   # keep the exported buffers alive until every peer is done
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [(2,) + CASES[0][1:], CASES[1]], ids=["top1", "top2"])
def test_ep_two_processes_through_cuda_ipc(case):
    import torch.multiprocessing as mp
    world = case[0]
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ipc_rank, args=(world, port, case, out), nprocs=world, start_method="spawn", join=True)
    assert all(out[g] for g in range(world)), dict(out)
