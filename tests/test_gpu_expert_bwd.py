"""Backward of the expert FFN on the tensor cores (moe_expert_backward)
through the C ABI against the oracle's expert-path backward (pinned by finite
differences in test_oracle_pins.py).  Needs a B200.

The routing, slot claim and gathered rows come from the library's own forward
calls (moe_route, moe_dispatch: integer routing is bit-exact with the oracle's,
tested elsewhere); the oracle then takes the same gates, drops and upstream
gradient.  Tolerance (bf16 operands -- dY, dU, the recomputed activations --
with fp32 accumulation): relative RMS <= 1e-2 per gradient tensor and the
per-element guard of the layer outputs, |got - ref| <= 3e-2 RMS(ref row) +
4e-3 |ref| (rows: an output row of dx or of a weight gradient).

ReLU's derivative is a decision floating point takes (u > 0).  The kernel
decides on its fp32-accumulated pre-activation, the oracle on its fp64 one;
where |u| is within 1e-5 of zero (~25x the fp32 accumulation error at these
shapes) the two may decide differently, and one flipped decision moves a
whole row of dx and of dW1 by one product term.  The per-element guard
therefore skips the tokens (dx) and the (expert, hidden unit) rows (dW1, db1)
that have such a near-zero pre-activation, found from the fp64 pre-activations
of the kept rows; the relative-RMS bound still covers every element."""
import concurrent.futures

import numpy as np
import pytest

import oracle
from gpu_helpers import assert_elementwise, host_threads, rel_rms
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.layer import to_device, to_host_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

CASES = [
    # T, d, d_ff, N, k, cf, act, biases, router bias (None, or "empty": four experts get no token)
    (2000, 256, 512, 8, 1, 1.25, "relu", False, None),
    (1500, 128, 384, 4, 2, 1.0, "swiglu", True, None),
    (3000, 192, 320, 6, 2, 1.25, "relu", True, None),
    (1200, 128, 256, 8, 1, 2.0, "relu", False, "empty"),
    (8192, 512, 1024, 16, 1, 1.25, "relu", False, None),     # several tiles per CTA in every GEMM
    (4096, 256, 512, 8, 2, 1.25, "swiglu", False, None),
]


def assert_grad_close(got, ref, what, skip_rows=None):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rr = rel_rms(got, ref)
    assert rr <= 1e-2, f"{what}: rel RMS {rr:.3e}"
    if skip_rows is not None:
        keep = ~np.asarray(skip_rows, bool)
        got, ref = got[keep], ref[keep]
    assert_elementwise(got, ref, what)


NEAR_ZERO = 1e-5


def relu_near_ties(L, idx, drop, N, act):
    """(tokens [T] bool, hidden units [N, d_ff] bool) whose kept rows have a
    pre-activation u = W1[e] x + b1 within NEAR_ZERO of 0 (fp64)."""
    T = idx.shape[0]
    d_ff = L["w1"].shape[1]
    tok = np.zeros(T, bool)
    unit = np.zeros((N, d_ff), bool)
    if act != "relu":
        return tok, unit
    x = oracle.widen(L["x"])
    w1 = oracle.widen(L["w1"])
    b1 = None if L["b1"] is None else oracle.widen(L["b1"])
    for e in range(N):
        t, r = np.nonzero((idx == e) & (drop == 0))
        if t.size == 0:
            continue
        u = x[t] @ w1[e].T
        if b1 is not None:
            u += b1[e]
        near = np.abs(u) < NEAR_ZERO
        tok[t[near.any(axis=1)]] = True
        unit[e] |= near.any(axis=0)
    return tok, unit


def _oracle_bwd(L, weights, idx, gate, drop, dout, act):
    """oracle.expert_backward over token chunks on host threads; the gradient
    sums of the chunks are added in fp64 (far below the bf16 tolerance)."""
    T = idx.shape[0]
    n = max(1, min(host_threads(), T // 256))
    bounds = np.linspace(0, T, n + 1).astype(int)

    def one(i):
        a, b = bounds[i], bounds[i + 1]
        return oracle.expert_backward(L["x"][a:b], weights, idx[a:b], gate[a:b], drop[a:b], dout[a:b], act)

    with concurrent.futures.ThreadPoolExecutor(max_workers=n) as ex:
        parts = list(ex.map(one, range(n)))
    out = {"dx": np.concatenate([p["dx"] for p in parts])}
    for key in ("dw1", "db1", "dw3", "db3", "dw2", "db2"):
        out[key] = None if parts[0][key] is None else sum(p[key] for p in parts)
    return out


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}_d{}_ff{}_N{}_k{}_{}".format(*c[:5], c[6]))
def test_expert_backward_matches_oracle(case):
    T, d, dff, N, k, cf, act, biases, rb = case
    router_bias = None
    if rb == "empty":
        router_bias = np.zeros(N, np.float32)
        router_bias[N // 2:] = -30.0
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype="bf16", biases=biases,
                          seed=T + 3 * N, router_bias=router_bias)
    C = nat.moe_capacity(T, N, k, cf)
    cfg = nat.config(T, d, dff, N, k, C, "bf16", act)
    ws = nat.new_workspace(cfg)
    dev = dict(device="cuda")
    R = max(1, min(k * T, N * C))
    x = to_device(L["x"])
    W = {key: to_device(L[key]) for key in ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")}
    idx = torch.empty(T, k, dtype=torch.int32, **dev)
    gate = torch.empty(T, k, dtype=torch.float32, **dev)
    pos = torch.empty(T, k, dtype=torch.int32, **dev)
    drop = torch.empty(T, k, dtype=torch.uint8, **dev)
    counts = torch.empty(k, N, dtype=torch.int32, **dev)
    kept = torch.empty(N, dtype=torch.int32, **dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, **dev)
    row_token = torch.empty(R, dtype=torch.int32, **dev)
    row_gate = torch.empty(R, dtype=torch.float32, **dev)
    xe = torch.empty(R, d, dtype=torch.bfloat16, **dev)
    nat.check(nat.moe_route(cfg, x, W["w_r"], W["b_r"], idx, gate, None, None, None, None, ws))
    nat.check(nat.moe_dispatch(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, ws))
    rng = np.random.default_rng(T)
    dout_h = oracle.bf16_bits((0.1 * rng.standard_normal((T, d))).astype(np.float32))
    dout = to_device(dout_h)
    nb = nat.moe_expert_backward_workspace_bytes(cfg)
    assert nb > 0
    wsb = torch.empty(nb, dtype=torch.uint8, **dev)
    nat.check(nat.moe_workspace_init(wsb))
    f32 = dict(dtype=torch.float32, **dev)
    sw = act == "swiglu"
    g = dict(dx=torch.full((T, d), float("nan"), **f32), dw1=torch.full((N, dff, d), float("nan"), **f32),
             db1=torch.full((N, dff), float("nan"), **f32) if biases else None,
             dw3=torch.full((N, dff, d), float("nan"), **f32) if sw else None,
             db3=torch.full((N, dff), float("nan"), **f32) if (sw and biases) else None,
             dw2=torch.full((N, d, dff), float("nan"), **f32),
             db2=torch.full((N, d), float("nan"), **f32) if biases else None)
    nat.check(nat.moe_expert_backward(cfg, xe, offsets, row_token, row_gate, idx, pos, drop, dout, W["w1"], W["b1"],
                                      W["w3"], W["b3"], W["w2"], g["dx"], g["dw1"], g["db1"], g["dw3"], g["db3"],
                                      g["dw2"], g["db2"], wsb))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(wsb))
    weights = {key: L[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    ref = _oracle_bwd(L, weights, idx.cpu().numpy(), gate.cpu().numpy(), drop.cpu().numpy(),
                      oracle.widen(dout_h).astype(np.float32), oracle.SWIGLU if sw else oracle.RELU)
    near_tok, near_unit = relu_near_ties(L, idx.cpu().numpy(), drop.cpu().numpy(), N, act)
    skip = {"dx": near_tok, "dw1": near_unit.reshape(-1), "db1": near_unit}
    for key, t in g.items():
        if t is None:
            continue
        got = t.cpu().numpy()
        assert np.isfinite(got).all(), f"{key}: not every element written"
        if key.startswith("dw"):
            for e in range(N):
                if not ref[key][e].any():
                    assert not got[e].any(), f"{key}[{e}]: an expert without rows must get zeros"
            assert_grad_close(got.reshape(-1, got.shape[-1]), ref[key].reshape(-1, got.shape[-1]), key,
                              skip.get(key))
        elif key == "db1":
            rr = rel_rms(got, ref[key])
            assert rr <= 1e-2, f"{key}: rel RMS {rr:.3e}"
            keep = ~near_unit
            assert_elementwise(got[keep].reshape(1, -1), ref[key][keep].reshape(1, -1), key)
        else:
            assert_grad_close(got, ref[key], key, skip.get(key))
    assert near_tok.mean() < 0.1, "too many near-zero pre-activations for a meaningful per-element check"
    if rb == "empty":
        assert not g["dw1"][N // 2:].any().item()
    # tokens with no kept assignment: dx exactly zero
    all_drop = drop.cpu().numpy().all(axis=1)
    assert not g["dx"].cpu().numpy()[all_drop].any()


def test_expert_backward_rejects_fp32():
    cfg = nat.config(100, 64, 64, 4, 1, 30, "f32")
    assert nat.moe_expert_backward_workspace_bytes(cfg) == 0
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    st = nat.moe_expert_backward(cfg, t, t, t, t, t, t, t, t, t, None, None, None, t, t, None, None, None, None, None,
                                 None, t)
    assert st == nat.MOE_ERR_UNSUPPORTED
