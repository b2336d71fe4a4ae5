"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare with the stated tolerances.

Tolerances (stated for the layer): integer routing outputs bit-exact; router
probabilities, gates, P_i and the aux loss within 1e-5 relative; bf16 layer
outputs within 2e-2 max-abs AND 1e-2 relative RMS (fp32 accumulation); fp32
layer outputs within 1e-4 max-abs.

Per-element guard (bf16): the layer's outputs are small (|out| ~ 1e-2 at
s = 0.1 init), so the 2e-2 max-abs bound alone passes a wrong element.  Every
element must also satisfy |got - ref| <= 3e-2 * RMS(ref row) + 4e-3 * |ref|.
The bf16 arithmetic explains at most ~2^-9 |ref| (the final rounding) plus
~1e-3 RMS per element of H's bf16 rounding propagated through W2 (a few times
that at the tail of a row's distribution); an element computed from the wrong
operand tile is off by about the row's RMS and fails.
"""
import concurrent.futures
import functools
import os

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
ELEM_ROW_RMS = 3e-2
ELEM_VALUE = 4e-3


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
    assert_elementwise(got, ref, what)


def assert_elementwise(got, ref, what="out"):
    """bf16 per-element guard: |got - ref| <= 3e-2 RMS(row of ref) + 4e-3 |ref|
    (an all-zero reference row must come back exactly zero)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return
    g2 = got.reshape(-1, ref.shape[-1]) if ref.ndim > 1 else got.reshape(1, -1)
    r2 = ref.reshape(g2.shape)
    rms = np.sqrt(np.mean(r2 * r2, axis=1, keepdims=True))
    bound = ELEM_ROW_RMS * rms + ELEM_VALUE * np.abs(r2)
    bad = np.abs(g2 - r2) > bound
    if bad.any():
        i, j = np.unravel_index(np.argmax(np.where(bad, np.abs(g2 - r2) / np.maximum(bound, 1e-300), 0)), bad.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements beyond the per-element guard; worst row {i} col {j}: "
                             f"got {g2[i, j]:.6e} ref {r2[i, j]:.6e} row RMS {rms[i, 0]:.3e}")


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


def host_threads():
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1))


def oracle_layer_threads(L, k, C, act, dtype, alpha=1e-2, tokens=None, chunk=64):
    """oracle.forward's result with the per-token expert work spread over host
    threads: routing, aux loss and the (serial) slot claim run once; the
    oracle's own single-threaded per-token function then evaluates disjoint
    token chunks side by side (each token's arithmetic is independent and
    sequential, so the values are those of one call)."""
    weights = {key: L[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    routing = oracle.route(L["x"], L["w_r"], L["b_r"], k)
    f, P, aux = oracle.aux_loss(routing["idx"], routing["probs"], alpha)
    N = np.asarray(L["w_r"]).shape[0]
    disp = oracle.dispatch(routing["idx"], N, C)
    T = np.asarray(L["x"]).shape[0]
    toks = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    out_dtype = oracle.BF16 if dtype == "bf16" else oracle.F32
    parts = [toks[i:i + chunk] for i in range(0, toks.size, chunk)] or [toks]

    def one(tk):
        return oracle.layer_tokens(L["x"], weights, routing, disp, tk, act_code(act), out_dtype)

    with concurrent.futures.ThreadPoolExecutor(max_workers=host_threads()) as ex:
        res = list(ex.map(one, parts))
    d = np.asarray(L["x"]).shape[1]
    out_exact = np.concatenate([r[0] for r in res]) if res else np.zeros((0, d))
    out_rounded = np.concatenate([r[1] for r in res]) if res else np.zeros((0, d), np.float32)
    return dict(routing=routing, f=f, P=P, aux=aux, disp=disp, tokens=toks, out_exact=out_exact, out=out_rounded)


def compact_rows(idx, disp):
    """Token and rank of every compact expert-major row (row = offsets[e] + pos)."""
    off, pos, drop = disp["offsets"], disp["pos"], disp["drop"]
    n = int(off[-1])
    row_token = np.full(n, -1, np.int64)
    row_expert = np.full(n, -1, np.int32)
    kt, kr = np.nonzero(drop == 0)
    rows = off[idx[kt, kr]] + pos[kt, kr]
    row_token[rows] = kt
    row_expert[rows] = idx[kt, kr]
    return row_token, row_expert


def tile_cover_tokens(idx, disp, block):
    """Tokens whose compact rows include, for every expert, its first row and the
    last valid row of every `block`-row slice of its rows: every m-tile of both
    expert GEMMs (tiles of `block` or a multiple of it), the last row of every
    ragged tile among them, has a checked row."""
    row_token, _ = compact_rows(idx, disp)
    off = disp["offsets"]
    rows = []
    for e in range(off.size - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi <= lo:
            continue
        rows.append(lo)
        rows.extend(range(min(lo + block, hi) - 1, hi, block))
        rows.append(hi - 1)
    return np.unique(row_token[np.asarray(rows, np.int64)])


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
