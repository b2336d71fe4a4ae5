"""Router backward through the C ABI (moe_router_backward) against the oracle:
dL/dh, dW_r, db_r and the router's part of dL/dx for L = sum dgate * gate +
L_aux (gate path of "From Switch Transformer to GLaM"; load-balancing
gradient through P with coefficient f, CMU 10-423 Lecture 16, section 4.2).
Inputs are the oracle's forward values (probs, idx, gate, f), so both sides
differentiate the same point.  bf16 layers take the tensor-core path (exact
three-way bf16 splits of dh and W_r, fp32 accumulation over token chunks,
fp64 over chunks), fp32 layers the FP32 pipe: tolerances are relative to each
output's largest magnitude.  Needs a B200."""
import numpy as np
import pytest

import oracle
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.layer import to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

TOL_DH = 2e-6   # per-token fp32 arithmetic over N terms
TOL_SUM = 1e-5  # fp32 sums over 512-token chunks


def _close(got, ref, tol, what):
    ref = np.asarray(ref, np.float64)
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(np.asarray(got, np.float64) - ref).max()) if ref.size else 0.0
    assert err <= tol * scale + 1e-12, f"{what}: max abs err {err:.3e} vs scale {scale:.3e}"


def _run(L, r, f, dgate, T, d, N, k, dtype, alpha):
    cfg = nat.config(T, d, 64, N, k, max(T, 1), dtype, "relu", alpha)
    ws = nat.new_workspace(cfg)
    dev = dict(device="cuda")
    out = dict(dh=torch.full((max(T, 1), N), np.nan, dtype=torch.float32, **dev),
               dw=torch.full((N, d), np.nan, dtype=torch.float32, **dev),
               db=torch.full((N,), np.nan, dtype=torch.float32, **dev),
               dx=torch.full((max(T, 1), d), np.nan, dtype=torch.float32, **dev))
    nat.check(nat.moe_router_backward(cfg, to_device(L["x"]), to_device(L["w_r"]), to_device(r["probs"]),
                                      to_device(r["idx"]), to_device(r["gate"]), to_device(f), to_device(dgate),
                                      out["dh"], out["dw"], out["db"], out["dx"], ws))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(ws))
    return {key: v.cpu().numpy() for key, v in out.items()}


@pytest.mark.parametrize("T,d,N,k,dtype", [(3000, 128, 8, 1, "bf16"), (2049, 256, 64, 2, "bf16"),
                                           (777, 64, 40, 2, "f32"), (4096, 128, 128, 1, "bf16"), (1, 64, 12, 1, "f32")])
def test_router_backward_matches_oracle(T, d, N, k, dtype):
    alpha = 0.01
    L = inputs.make_layer(T=T, d_model=d, d_ff=64, n_experts=N, top_k=k, dtype=dtype, seed=T + N,
                          router_bias=np.linspace(0.4, 0.0, N).astype(np.float32))
    r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
    f, _, _ = oracle.aux_loss(r["idx"], r["probs"], alpha)
    dgate = np.random.default_rng(T).standard_normal((T, k)).astype(np.float32)
    ref = oracle.router_backward(L["x"], L["w_r"], r["probs"], r["idx"], r["gate"], f, dgate, alpha)
    got = _run(L, r, f, dgate, T, d, N, k, dtype, alpha)
    _close(got["dh"], ref["dh"], TOL_DH, "dh")
    _close(got["dw"], ref["dw"], TOL_SUM, "dW_r")
    _close(got["db"], ref["db"], TOL_SUM, "db_r")
    _close(got["dx"], ref["dx"], TOL_SUM, "dx")
    again = _run(L, r, f, dgate, T, d, N, k, dtype, alpha)
    for key in got:
        np.testing.assert_array_equal(got[key], again[key], err_msg=f"{key} not deterministic")


def test_router_backward_full_size_matches_oracle():
    # the Switch-Base router at full size: T = 65536 tokens, d = 768, N = 64,
    # top-1, bf16 tokens: every output element against the oracle
    T, d, N, k, alpha = 65536, 768, 64, 1, 0.01
    L = inputs.make_layer(T=T, d_model=d, d_ff=64, n_experts=N, top_k=k, dtype="bf16", seed=65)
    r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
    f, _, _ = oracle.aux_loss(r["idx"], r["probs"], alpha)
    dgate = np.random.default_rng(65).standard_normal((T, k)).astype(np.float32)
    ref = oracle.router_backward(L["x"], L["w_r"], r["probs"], r["idx"], r["gate"], f, dgate, alpha)
    got = _run(L, r, f, dgate, T, d, N, k, "bf16", alpha)
    _close(got["dh"], ref["dh"], TOL_DH, "dh")
    _close(got["dw"], ref["dw"], TOL_SUM, "dW_r")
    _close(got["db"], ref["db"], TOL_SUM, "db_r")
    _close(got["dx"], ref["dx"], TOL_SUM, "dx")


def test_router_backward_empty_batch():
    L = inputs.make_layer(T=0, d_model=64, d_ff=64, n_experts=8, top_k=1, dtype="bf16", seed=1)
    r = dict(probs=np.zeros((0, 8), np.float32), idx=np.zeros((0, 1), np.int32), gate=np.zeros((0, 1), np.float32))
    got = _run(L, r, np.zeros(8), np.zeros((0, 1), np.float32), 0, 64, 8, 1, "bf16", 0.01)
    assert np.all(got["dw"] == 0) and np.all(got["db"] == 0)


def test_router_backward_time_at_switch_base_size():
    # T = 65536, d = 768, N = 64, top-1 (reported, not asserted beyond completion)
    T, d, N = 65536, 768, 64
    rng = np.random.default_rng(6)
    h = rng.standard_normal((T, N)).astype(np.float32)
    p = np.exp(h - h.max(axis=1, keepdims=True))
    probs = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    idx = np.argmax(probs, axis=1).astype(np.int32)[:, None]
    gate = probs[np.arange(T), idx[:, 0]][:, None].copy()
    cfg = nat.config(T, d, 3072, N, 1, 1280)
    ws = nat.new_workspace(cfg)
    dev = dict(device="cuda")
    args = [cfg, to_device(rng.integers(0, 1 << 14, size=(T, d)).astype(np.uint16)),
            to_device((rng.standard_normal((N, d)) * 0.01).astype(np.float32)), to_device(probs), to_device(idx),
            to_device(gate), to_device(np.full(N, 1.0 / N)), to_device(rng.standard_normal((T, 1)).astype(np.float32)),
            torch.empty(T, N, dtype=torch.float32, **dev), torch.empty(N, d, dtype=torch.float32, **dev),
            torch.empty(N, dtype=torch.float32, **dev), torch.empty(T, d, dtype=torch.float32, **dev), ws]
    nat.check(nat.moe_router_backward(*args))
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(10):
        nat.check(nat.moe_router_backward(*args))
    ev[1].record()
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(ws))
    print(f"\nrouter backward at T={T}, d={d}, N={N}: {ev[0].elapsed_time(ev[1]) / 10 * 1e3:.1f} us")
