"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare with the stated tolerances.

Tolerances (stated for the layer): integer routing outputs bit-exact; router
probabilities, gates, P_i and the aux loss within 1e-5 relative; bf16 layer
outputs within 2e-2 max-abs AND 1e-2 relative RMS (fp32 accumulation); fp32
layer outputs within 1e-4 max-abs.
"""
import functools

import numpy as np

import oracle
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.configs import WORKLOADS
from mixture_experts_sparse_b200.layer import MoeLayer, to_device, to_host_bits

REL_PROB = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_RMS = 1e-2
F32_MAX_ABS = 1e-4


def widen_out(t):
    """device output -> fp64 numpy values"""
    return oracle.widen(to_host_bits(t))


def rel_rms(a, ref):
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    num = np.sqrt(np.mean((a - ref) ** 2)) if ref.size else 0.0
    return num / den if den > 0 else num


def assert_close_out(got, ref, dtype, what="out"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return
    err = np.abs(got - ref).max()
    if dtype == "f32":
        assert err <= F32_MAX_ABS, f"{what}: max abs {err:.3e} > {F32_MAX_ABS}"
        return
    assert err <= BF16_MAX_ABS, f"{what}: max abs {err:.3e} > {BF16_MAX_ABS}"
    if np.any(ref != 0):
        rr = rel_rms(got, ref)
        assert rr <= BF16_REL_RMS, f"{what}: rel RMS {rr:.3e} > {BF16_REL_RMS}"
    else:
        assert np.all(got == 0), f"{what}: expected exact zeros"


def assert_rel(got, ref, tol, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bad = np.abs(got - ref) > tol * np.abs(ref) + 1e-30
    assert not bad.any(), f"{what}: {bad.sum()} values beyond {tol} relative, worst at {np.argmax(np.abs(got-ref))}"


@functools.lru_cache(maxsize=2)
def workload_inputs(name, **over):
    w = WORKLOADS[name]
    return inputs.make_workload(w, **over)


def act_code(act):
    return oracle.SWIGLU if act == "swiglu" else oracle.RELU


def run_layer(L, T, d, d_ff, N, k, C, dtype, act, alpha=1e-2):
    """moe_forward on the GPU with every routing output requested."""
    import torch
    layer = MoeLayer(T, d, d_ff, N, k, C, dtype, act, L, alpha=alpha)
    x = to_device(L["x"])
    nat.check(layer.forward(x))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(layer.ws))
    return layer, x


def oracle_layer(L, k, C, act, dtype, alpha=1e-2, tokens=None):
    weights = {key: L[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    return oracle.forward(L["x"], L["w_r"], L["b_r"], weights, k=k, C=C, act=act_code(act), alpha=alpha,
                          out_dtype=oracle.BF16 if dtype == "bf16" else oracle.F32, tokens=tokens)


def compare_routing(layer, res):
    r, dd = res["routing"], res["disp"]
    np.testing.assert_array_equal(layer.idx.cpu().numpy(), r["idx"], err_msg="idx")
    assert_rel(layer.gate.cpu().numpy(), r["gate"], REL_PROB, "gate")
    np.testing.assert_array_equal(layer.pos.cpu().numpy(), dd["pos"], err_msg="pos")
    np.testing.assert_array_equal(layer.drop.cpu().numpy(), dd["drop"], err_msg="drop")
    np.testing.assert_array_equal(layer.counts.cpu().numpy(), dd["counts"], err_msg="counts")
    np.testing.assert_array_equal(layer.kept.cpu().numpy(), dd["kept"], err_msg="kept")
    np.testing.assert_array_equal(layer.offsets.cpu().numpy(), dd["offsets"], err_msg="offsets")
    np.testing.assert_array_equal(layer.f.cpu().numpy(), res["f"], err_msg="f")
    assert_rel(layer.P.cpu().numpy(), res["P"], REL_PROB, "P")
    assert_rel(layer.aux.cpu().numpy()[0], res["aux"], REL_PROB, "aux")


def sample_tokens(T, drop, n_random=24, seed=0):
    """first/last tokens, random ones, and dropped / partially dropped tokens"""
    rng = np.random.default_rng(seed)
    picks = set(range(min(8, T))) | set(range(max(0, T - 8), T))
    if T > 0:
        picks |= set(rng.integers(0, T, size=n_random).tolist())
    all_drop = np.nonzero(drop.all(axis=1))[0]
    some_drop = np.nonzero(drop.any(axis=1) & ~drop.all(axis=1))[0]
    picks |= set(all_drop[:6].tolist()) | set(all_drop[-2:].tolist()) | set(some_drop[:6].tolist())
    return np.array(sorted(picks), dtype=np.int64)
