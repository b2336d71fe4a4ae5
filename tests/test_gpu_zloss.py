"""Router z-loss through the C ABI (moe_route_z) against the oracle's
definition (CMU 10-423 Lecture 16, section 4.2, read as the mean over tokens
of the squared log-sum-exp of the router logits), on both router paths:
the tensor-core router (bf16 input, expert counts padded to 32/64/128) and
the FP32-pipe router (fp32 input).  The other router outputs must be the
same bits as moe_route's.  Needs a B200."""
import numpy as np
import pytest

import oracle
from gpu_helpers import REL_PROB, assert_rel
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.layer import to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

CASES = [  # T, d, N, k, dtype, router bias
    (5000, 128, 8, 1, "bf16", False),
    (4097, 256, 64, 2, "bf16", True),
    (3000, 128, 128, 1, "bf16", True),
    (1, 64, 12, 2, "bf16", True),
    (777, 64, 8, 1, "f32", True),
    (1500, 96, 40, 2, "f32", False),
]


def _route(L, T, d, N, k, dtype, with_z):
    cfg = nat.config(T, d, 64, N, k, max(1, T), dtype, "relu")
    ws = nat.new_workspace(cfg)
    dev = dict(device="cuda")
    out = dict(idx=torch.full((max(T, 1), k), -1, dtype=torch.int32, **dev),
               gate=torch.full((max(T, 1), k), -1.0, dtype=torch.float32, **dev),
               probs=torch.full((max(T, 1), N), -1.0, dtype=torch.float32, **dev),
               f=torch.full((N,), -1.0, dtype=torch.float64, **dev),
               P=torch.full((N,), -1.0, dtype=torch.float64, **dev),
               aux=torch.full((1,), -1.0, dtype=torch.float64, **dev),
               z=torch.full((1,), -1.0, dtype=torch.float64, **dev))
    x, w_r, b_r = to_device(L["x"]), to_device(L["w_r"]), to_device(L["b_r"])
    if with_z:
        nat.check(nat.moe_route_z(cfg, x, w_r, b_r, out["idx"], out["gate"], out["probs"], out["f"], out["P"],
                                  out["aux"], out["z"], ws))
    else:
        nat.check(nat.moe_route(cfg, x, w_r, b_r, out["idx"], out["gate"], out["probs"], out["f"], out["P"],
                                out["aux"], ws))
    torch.cuda.synchronize()
    assert nat.moe_read_device_status(ws) == nat.MOE_OK
    return {key: v.cpu().numpy() for key, v in out.items()}


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_N%d_k%d_%s%s" % (c[0], c[1], c[2], c[3], c[4],
                                                                               "_bias" if c[5] else ""))
def test_route_z_matches_oracle(case):
    T, d, N, k, dtype, bias = case
    rb = np.linspace(0.3, -0.2, N).astype(np.float32) if bias else None
    L = inputs.make_layer(T=T, d_model=d, d_ff=64, n_experts=N, top_k=k, dtype=dtype, seed=T + N, router_bias=rb)
    r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
    got = _route(L, T, d, N, k, dtype, True)
    assert_rel(got["z"][0], oracle.z_loss(r["logits"]), REL_PROB, "z-loss")
    plain = _route(L, T, d, N, k, dtype, False)
    for key in ("idx", "gate", "probs", "f", "P", "aux"):
        np.testing.assert_array_equal(got[key], plain[key], err_msg=key)


def test_route_z_empty_batch():
    L = inputs.make_layer(T=0, d_model=64, d_ff=64, n_experts=8, top_k=1, dtype="bf16", seed=1)
    got = _route(L, 0, 64, 8, 1, "bf16", True)
    assert got["z"][0] == 0.0
