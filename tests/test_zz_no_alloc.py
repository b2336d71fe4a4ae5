"""moe_dispatch_noalloc -- the dispatch for callers that cannot allocate device
memory when they call the layer (plugin interfaces that receive only their
input and output tensors; serving runtimes that reserve all device memory at
start-up and allow no cudaMalloc later).  Its scratch lives in a fixed-size
array inside the library instead of a caller workspace.

Checked through the C ABI on two calls in a row (the shared array keeps the
previous call's contents, so the second call shows that each call clears what
it uses), against the oracle's slot claim and against moe_dispatch with a
workspace: integer outputs, row maps and gathered rows must be identical (the
tolerance the parity tests use for integer and copy work).  One case fills the
array exactly (the largest T, top-2, 128 experts).  This file is collected
last on purpose."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from mixture_experts_sparse_b200 import inputs  # noqa: E402
from mixture_experts_sparse_b200 import native as nat  # noqa: E402
from mixture_experts_sparse_b200.layer import to_device, to_host_bits  # noqa: E402

import oracle  # noqa: E402


def _buffers(T, k, N, R, d):
    z = dict(device="cuda")
    return dict(pos=torch.full((T, k), -7, dtype=torch.int32, **z),
                drop=torch.full((T, k), 9, dtype=torch.uint8, **z),
                counts=torch.full((k, N), -7, dtype=torch.int32, **z),
                kept=torch.full((N,), -7, dtype=torch.int32, **z),
                offsets=torch.full((N + 1,), -7, dtype=torch.int32, **z),
                row_token=torch.full((R,), -7, dtype=torch.int32, **z),
                row_gate=torch.full((R,), -7.0, dtype=torch.float32, **z),
                xe=torch.zeros(R, d, dtype=torch.bfloat16, **z))


def _oracle_rows(idx, gate, dd, T, k):
    nrows = int(dd["offsets"][-1])
    want_t = np.full(nrows, -1, np.int32)
    want_g = np.zeros(nrows, np.float32)
    kt, kr = np.nonzero(dd["drop"] == 0)
    rows = dd["offsets"][idx[kt, kr]] + dd["pos"][kt, kr]
    want_t[rows] = kt
    want_g[rows] = gate[kt, kr]
    return want_t, want_g


def _run_case(T, d, N, k, C, idx_h, gate_h, x_h):
    cfg = nat.config(T, d, 64, N, k, C)
    R = max(1, min(k * T, N * C))
    x, idx, gate = to_device(x_h), to_device(idx_h), to_device(gate_h)
    dd = oracle.dispatch(idx_h, N, C)
    want_t, want_g = _oracle_rows(idx_h, gate_h, dd, T, k)
    nrows = want_t.size

    ref = _buffers(T, k, N, R, d)
    ws = nat.new_workspace(cfg)
    nat.check(nat.moe_dispatch(cfg, x, idx, gate, ref["pos"], ref["drop"], ref["counts"], ref["kept"],
                               ref["offsets"], ref["row_token"], ref["row_gate"], ref["xe"], ws))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(ws))

    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        got = _buffers(T, k, N, R, d)
        nat.check(nat.moe_dispatch_noalloc(cfg, x, idx, gate, got["pos"], got["drop"], got["counts"],
                                           got["kept"], got["offsets"], got["row_token"], got["row_gate"],
                                           got["xe"], status))
        torch.cuda.synchronize()
        assert status.item() == nat.MOE_OK, f"call {call}: device status {status.item()}"
        # the oracle's slot claim
        for key in ("pos", "drop", "counts", "kept", "offsets"):
            np.testing.assert_array_equal(got[key].cpu().numpy(), dd[key], err_msg=f"call {call}: {key} vs oracle")
        np.testing.assert_array_equal(got["row_token"].cpu().numpy()[:nrows], want_t, err_msg=f"call {call}")
        np.testing.assert_array_equal(got["row_gate"].cpu().numpy()[:nrows], want_g, err_msg=f"call {call}")
        np.testing.assert_array_equal(to_host_bits(got["xe"])[:nrows], x_h[want_t], err_msg=f"call {call}")
        # the workspace dispatch, every output buffer
        for key in ("pos", "drop", "counts", "kept", "offsets", "row_token", "row_gate"):
            np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key].cpu().numpy(),
                                          err_msg=f"call {call}: {key}")
        np.testing.assert_array_equal(to_host_bits(got["xe"]), to_host_bits(ref["xe"]))


@pytest.mark.parametrize("k", [1, 2])
def test_dispatch_noalloc_matches_oracle_and_workspace_dispatch(k):
    T, d, N = 5000, 128, 12
    L = inputs.make_layer(T=T, d_model=d, d_ff=64, n_experts=N, top_k=k, dtype="bf16", seed=41 + k,
                          router_bias=np.linspace(0.5, 0.0, N).astype(np.float32))
    r = oracle.route(L["x"], L["w_r"], L["b_r"], k)          # routing input, from the oracle
    C = nat.moe_capacity(T, N, k, 1.0)
    _run_case(T, d, N, k, C, r["idx"], r["gate"], L["x"])


def test_dispatch_noalloc_fills_the_whole_array():
    # T = 2^18, top-2, 128 experts: 256 scan blocks x 2 x 128 look-back words,
    # exactly the array's size.  Synthetic top-2 choices (two distinct experts
    # per token, skewed towards the low indices) and gates.
    T, d, N, k = 1 << 18, 16, 128, 2
    rng = np.random.default_rng(5)
    e0 = np.minimum((rng.exponential(24.0, T)).astype(np.int64), N - 1)
    e1 = (e0 + 1 + rng.integers(0, N - 1, T)) % N
    idx = np.stack([e0, e1], axis=1).astype(np.int32)
    gate = rng.random((T, k)).astype(np.float32)
    x = rng.integers(0, 1 << 15, size=(T, d)).astype(np.uint16)
    C = nat.moe_capacity(T, N, k, 1.0)
    _run_case(T, d, N, k, C, idx, gate, x)


def test_dispatch_noalloc_empty_batch_with_null_outputs():
    T, N, k = 0, 8, 2
    cfg = nat.config(T, 128, 64, N, k, 10)
    z = dict(device="cuda")
    counts = torch.full((k, N), -7, dtype=torch.int32, **z)
    kept = torch.full((N,), -7, dtype=torch.int32, **z)
    offsets = torch.full((N + 1,), -7, dtype=torch.int32, **z)
    nat.check(nat.moe_dispatch_noalloc(cfg, None, None, None, None, None, counts, kept, offsets, None, None, None,
                                       None))
    torch.cuda.synchronize()
    assert not counts.any().item() and not kept.any().item() and not offsets.any().item()


def test_dispatch_noalloc_rejects_too_many_tokens():
    T = (1 << 18) + 1
    cfg = nat.config(T, 128, 64, 8, 1, 100)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = nat.moe_dispatch_noalloc(cfg, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy, dummy,
                                  None, None)
    assert st == nat.MOE_ERR_UNSUPPORTED
