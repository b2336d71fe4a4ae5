"""The seeded input generator honours its recipe (no GPU)."""
import numpy as np

from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200.configs import WORKLOADS


def test_generator_is_seeded_and_guarded():
    a = inputs.make_layer(T=700, d_model=64, d_ff=128, n_experts=16, top_k=2, dtype="bf16", seed=3)
    b = inputs.make_layer(T=700, d_model=64, d_ff=128, n_experts=16, top_k=2, dtype="bf16", seed=3)
    for key in ("x", "w_r", "w1", "w2"):
        np.testing.assert_array_equal(a[key], b[key])
    assert a["x"].dtype == np.uint16 and a["w1"].dtype == np.uint16 and a["w_r"].dtype == np.float32
    x = inputs.bf16_to_f32(a["x"]).astype(np.float64)
    h = x @ a["w_r"].astype(np.float64).T
    top = -np.sort(-h, axis=1)
    assert np.all(top[:, 0] - top[:, 1] >= inputs.GAP)
    assert np.all(top[:, 1] - top[:, 2] >= inputs.GAP)
    # LayerNormed rows (before the bf16 cast): mean 0, variance 1
    assert np.abs(x.mean(1)).max() < 1e-2 and np.abs(x.var(1) - 1).max() < 2e-2


def test_truncated_normal_scale():
    L = inputs.make_layer(T=8, d_model=128, d_ff=256, n_experts=4, dtype="f32", biases=True, seed=1)
    for key, fan_in in (("w_r", 128), ("w1", 128), ("w2", 256), ("b1", 128), ("b2", 256)):
        w = L[key].astype(np.float64)
        sigma = np.sqrt(0.1 / fan_in)
        assert np.abs(w).max() <= 2 * sigma * (1 + 1e-6)
        # std of a N(0, s^2) truncated at 2s is 0.8796 s
        assert abs(w.std() / sigma - 0.8796) < 0.05


def test_zipf_router_bias_and_rms():
    b = inputs.zipf_router_bias(128, 1.2)
    pop = np.exp(b / 3.0)
    assert abs(pop.sum() - 1) < 1e-5 and abs(pop[0] - 0.270) < 5e-3
    assert np.all(np.diff(b) < 0)
    L = inputs.make_layer(T=64, d_model=256, d_ff=64, n_experts=8, top_k=2, act="swiglu",
                          norm="rmsnorm", dtype="bf16", seed=2)
    x = inputs.bf16_to_f32(L["x"]).astype(np.float64)
    assert np.abs(np.sqrt((x * x).mean(1)) - 1).max() < 1e-2
    assert L["w3"] is not None and L["w3"].shape == (8, 64, 256)


def test_workload_table():
    assert [w for w in WORKLOADS] == ["tiny_f32", "switch_base", "top2", "skew", "mixtral"]
    m = WORKLOADS["mixtral"]
    assert (m.T, m.d_model, m.d_ff, m.n_experts, m.top_k, m.act) == (16384, 4096, 14336, 8, 2, "swiglu")
