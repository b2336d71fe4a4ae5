"""dL/dgate through the C ABI (moe_gate_grad) against the oracle's expert-path
backward: dgate[t, r] = <dL/dout_t, E_e(x_t)> for a kept assignment, 0 for a
dropped one (out_t = sum_r gate_{t,r} E(x_t), "From Switch Transformer to
GLaM").  The GPU reads the oracle's own expert rows rounded to the activation
dtype; the oracle uses them unrounded, so the bf16 tolerance is the layer
output's (2e-2 of the largest |dgate|), fp32 1e-4.  Needs a B200."""
import numpy as np
import pytest

import oracle
from gpu_helpers import act_code
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.layer import to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.mark.parametrize("T,d,dff,N,k,cf,act,dtype", [(2000, 128, 384, 6, 2, 1.0, "relu", "bf16"),
                                                      (1500, 192, 320, 4, 2, 1.25, "swiglu", "bf16"),
                                                      (512, 64, 256, 8, 1, 0.5, "relu", "f32")])
def test_gate_grad_matches_oracle(T, d, dff, N, k, cf, act, dtype):
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, seed=13,
                          biases=(dtype == "f32"))
    C = nat.moe_capacity(T, N, k, cf)
    r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
    dd = oracle.dispatch(r["idx"], N, C)
    weights = {key: L[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    rng = np.random.default_rng(T)
    dout32 = (rng.standard_normal((T, d)) * 0.5).astype(np.float32)
    dout = oracle.bf16_bits(dout32).reshape(T, d) if dtype == "bf16" else dout32
    dout_vals = oracle.widen(dout).astype(np.float32) if dtype == "bf16" else dout32
    ref = oracle.expert_backward(L["x"], weights, r["idx"], r["gate"], dd["drop"], dout_vals, act=act_code(act))
    nrows = int(dd["offsets"][-1])
    rows_token = np.zeros(nrows, np.int64)
    rows_expert = np.zeros(nrows, np.int32)
    kept = np.argwhere(dd["drop"] == 0)
    rows = dd["offsets"][r["idx"][kept[:, 0], kept[:, 1]]] + dd["pos"][kept[:, 0], kept[:, 1]]
    rows_token[rows] = kept[:, 0]
    rows_expert[rows] = r["idx"][kept[:, 0], kept[:, 1]]
    ye = oracle.expert_rows(L["x"], weights, rows_token, rows_expert, act_code(act))
    ye_in = oracle.bf16_bits(ye.astype(np.float32)).reshape(nrows, d) if dtype == "bf16" else ye.astype(np.float32)
    cfg = nat.config(T, d, dff, N, k, C, dtype, act)
    dgate = torch.full((T, k), np.nan, dtype=torch.float32, device="cuda")
    nat.check(nat.moe_gate_grad(cfg, to_device(dout), to_device(ye_in), to_device(r["idx"]), to_device(dd["pos"]),
                                to_device(dd["drop"]), to_device(dd["offsets"]), dgate))
    torch.cuda.synchronize()
    got = dgate.cpu().numpy().astype(np.float64)
    assert np.all(got[dd["drop"] == 1] == 0.0)
    tol = 2e-2 if dtype == "bf16" else 1e-4
    scale = float(np.abs(ref["dgate"]).max())
    err = float(np.abs(got - ref["dgate"]).max())
    assert err <= tol * scale, f"dgate: max abs err {err:.3e}, scale {scale:.3e}"
