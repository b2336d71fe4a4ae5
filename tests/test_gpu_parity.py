"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same
seeded inputs.  Needs a B200."""
import numpy as np
import pytest

import oracle
from gpu_helpers import (BF16_MAX_ABS, REL_PROB, act_code, assert_close_out, assert_rel, compare_routing,
                         oracle_layer, oracle_layer_threads, rel_rms, run_layer, sample_tokens, tile_cover_tokens,
                         widen_out, workload_inputs)
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.configs import WORKLOADS
from mixture_experts_sparse_b200.layer import to_device, to_host_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


# Small layers the oracle evaluates completely.  They span several m-tiles per
# expert with ragged tails, partial n-tiles (d_ff not a multiple of 256 / 128),
# non-power-of-two expert counts, biases, both activations and both dtypes.
SMALL = [
    # T,    d,   d_ff, N,  k, cf,   act,      dtype,  biases
    (3000, 256, 512, 8, 1, 1.25, "relu", "bf16", False),
    (2000, 128, 384, 6, 2, 1.0, "relu", "bf16", False),
    (1500, 192, 320, 4, 2, 1.25, "swiglu", "bf16", False),
    (1000, 128, 256, 8, 1, 1.0, "relu", "bf16", True),
    (900, 64, 192, 5, 2, 1.5, "swiglu", "bf16", True),
    (700, 96, 160, 16, 1, 2.0, "relu", "f32", True),
    (512, 64, 256, 8, 1, 1.0, "relu", "f32", True),
    (600, 48, 80, 3, 2, 1.0, "swiglu", "f32", False),
    (130, 128, 128, 128, 1, 4.0, "relu", "bf16", False),
    (257, 128, 256, 33, 2, 1.0, "relu", "bf16", False),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "T{}_d{}_ff{}_N{}_k{}_{}_{}".format(*c[:5], c[6], c[7]))
def test_forward_small_full_oracle(case):
    T, d, dff, N, k, cf, act, dtype, biases = case
    C = nat.moe_capacity(T, N, k, cf)
    assert C == oracle.capacity(T, N, k, cf)
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, biases=biases,
                          seed=T + N)
    layer, _ = run_layer(L, T, d, dff, N, k, C, dtype, act)
    res = oracle_layer(L, k, C, act, dtype)
    compare_routing(layer, res)
    assert_close_out(widen_out(layer.out), res["out_exact"], dtype)


def _route_inputs(case, seed=0):
    T, d, dff, N, k, cf, act, dtype, biases = case
    return inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, biases=biases,
                             seed=seed)


@pytest.mark.parametrize("case", SMALL[:3] + SMALL[5:7], ids=lambda c: f"N{c[3]}_k{c[4]}_{c[7]}")
def test_route_probs(case):
    T, d, dff, N, k, cf, act, dtype, biases = case
    L = _route_inputs(case, seed=5)
    C = nat.moe_capacity(T, N, k, cf)
    cfg = nat.config(T, d, dff, N, k, C, dtype, act)
    ws = nat.new_workspace(cfg)
    x = to_device(L["x"])
    w_r = to_device(L["w_r"])
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    probs = torch.empty(T, N, dtype=torch.float32, device="cuda")
    f = torch.empty(N, dtype=torch.float64, device="cuda")
    P = torch.empty(N, dtype=torch.float64, device="cuda")
    aux = torch.empty(1, dtype=torch.float64, device="cuda")
    nat.check(nat.moe_route(cfg, x, w_r, None, idx, gate, probs, f, P, aux, ws))
    torch.cuda.synchronize()
    r = oracle.route(L["x"], L["w_r"], None, k)
    fo, Po, auxo = oracle.aux_loss(r["idx"], r["probs"])
    np.testing.assert_array_equal(idx.cpu().numpy(), r["idx"])
    assert_rel(gate.cpu().numpy(), r["gate"], REL_PROB, "gate")
    assert_rel(probs.cpu().numpy(), r["probs"], REL_PROB, "probs")
    np.testing.assert_array_equal(f.cpu().numpy(), fo)
    assert_rel(P.cpu().numpy(), Po, REL_PROB, "P")
    assert_rel(aux.cpu().numpy()[0], auxo, REL_PROB, "aux")


@pytest.mark.parametrize("copy", [True, False], ids=["copy", "rowmap"])
@pytest.mark.parametrize("k", [1, 2])
@pytest.mark.parametrize("C", [0, 1, 37, 5000])
def test_dispatch_exact_from_oracle_routing(k, C, copy):
    # copy=False: no compact copy requested (xe = null), the row map alone
    T, d, N = 4099, 128, 7
    L = inputs.make_layer(T=T, d_model=d, d_ff=64, n_experts=N, top_k=k, dtype="bf16", seed=11,
                          router_bias=np.linspace(0.6, 0.0, N).astype(np.float32))
    r = oracle.route(L["x"], L["w_r"], L["b_r"], k)
    dd = oracle.dispatch(r["idx"], N, C)
    cfg = nat.config(T, d, 64, N, k, C)
    ws = nat.new_workspace(cfg)
    R = max(1, min(k * T, N * C))
    x = to_device(L["x"])
    idx = to_device(r["idx"])
    gate = to_device(r["gate"])
    pos = torch.empty(T, k, dtype=torch.int32, device="cuda")
    drop = torch.empty(T, k, dtype=torch.uint8, device="cuda")
    counts = torch.empty(k, N, dtype=torch.int32, device="cuda")
    kept = torch.empty(N, dtype=torch.int32, device="cuda")
    offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    row_token = torch.full((R,), -1, dtype=torch.int32, device="cuda")
    row_gate = torch.empty(R, dtype=torch.float32, device="cuda")
    xe = torch.zeros(R, d, dtype=torch.bfloat16, device="cuda") if copy else None
    nat.check(nat.moe_dispatch(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, ws))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(ws))
    np.testing.assert_array_equal(pos.cpu().numpy(), dd["pos"])
    np.testing.assert_array_equal(drop.cpu().numpy(), dd["drop"])
    np.testing.assert_array_equal(counts.cpu().numpy(), dd["counts"])
    np.testing.assert_array_equal(kept.cpu().numpy(), dd["kept"])
    np.testing.assert_array_equal(offsets.cpu().numpy(), dd["offsets"])
    nrows = int(dd["offsets"][-1])
    rt = row_token.cpu().numpy()[:nrows]
    rg = row_gate.cpu().numpy()[:nrows]
    want_t = np.full(nrows, -1)
    want_g = np.zeros(nrows, np.float32)
    for t in range(T):
        for rr in range(k):
            if not dd["drop"][t, rr]:
                row = dd["offsets"][r["idx"][t, rr]] + dd["pos"][t, rr]
                want_t[row] = t
                want_g[row] = r["gate"][t, rr]
    np.testing.assert_array_equal(rt, want_t)
    np.testing.assert_array_equal(rg, want_g)
    if copy:
        xe_h = to_host_bits(xe)[:nrows]
        np.testing.assert_array_equal(xe_h, L["x"][rt])


@pytest.mark.parametrize("case", [SMALL[0], SMALL[2], SMALL[6]], ids=lambda c: f"{c[6]}_{c[7]}")
def test_expert_ffn_and_combine_from_oracle_intermediates(case):
    T, d, dff, N, k, cf, act, dtype, biases = case
    L = _route_inputs(case, seed=21)
    C = nat.moe_capacity(T, N, k, cf)
    res = oracle_layer(L, k, C, act, dtype)
    r, dd = res["routing"], res["disp"]
    nrows = int(dd["offsets"][-1])
    rows_token = np.zeros(nrows, np.int64)
    rows_expert = np.zeros(nrows, np.int32)
    for t in range(T):
        for rr in range(k):
            if not dd["drop"][t, rr]:
                e = r["idx"][t, rr]
                row = dd["offsets"][e] + dd["pos"][t, rr]
                rows_token[row] = t
                rows_expert[row] = e
    weights = {key: L[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    ye_ref = oracle.expert_rows(L["x"], weights, rows_token, rows_expert, act_code(act))
    cfg = nat.config(T, d, dff, N, k, C, dtype, act)
    ws = nat.new_workspace(cfg)
    R = max(1, min(k * T, N * C))
    xe_h = np.zeros((R, d), L["x"].dtype)
    xe_h[:nrows] = L["x"][rows_token]
    xe = to_device(xe_h)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ye = torch.zeros(R, d, dtype=tdt, device="cuda")
    W = {key: to_device(L[key]) for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    offsets = to_device(dd["offsets"])
    nat.check(nat.moe_expert_ffn(cfg, xe, offsets, W["w1"], W["b1"], W["w3"], W["b3"], W["w2"], W["b2"], ye, ws))
    torch.cuda.synchronize()
    nat.check(nat.moe_read_device_status(ws))
    ye_got = widen_out(ye)[:nrows]
    assert_close_out(ye_got, ye_ref, dtype, "ye")
    # combine: the oracle's own expert rows, in the activation dtype, through moe_combine
    if dtype == "bf16":
        ye_in = to_device(oracle.bf16_bits(ye_ref.astype(np.float32)).reshape(nrows, d))
    else:
        ye_in = to_device(ye_ref.astype(np.float32))
    out = torch.empty(T, d, dtype=tdt, device="cuda")
    nat.check(nat.moe_combine(cfg, ye_in, to_device(r["idx"]), to_device(dd["pos"]), to_device(dd["drop"]),
                              to_device(r["gate"]), offsets, out))
    torch.cuda.synchronize()
    assert_close_out(widen_out(out), res["out_exact"], dtype, "combine")


# ------------------------------------------------------------ edge cases ----

def _edge(T, d, dff, N, k, C, act="relu", dtype="bf16", router_bias=None, seed=3, w_r_zero=False):
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, seed=seed,
                          router_bias=router_bias, gap_guard=not w_r_zero)
    if w_r_zero:
        L["w_r"] = np.zeros_like(L["w_r"])
    layer, _ = run_layer(L, T, d, dff, N, k, C, dtype, act)
    res = oracle_layer(L, k, C, act, dtype)
    compare_routing(layer, res)
    got = widen_out(layer.out)
    assert_close_out(got, res["out_exact"], dtype)
    return layer, res, got


@pytest.mark.parametrize("k", [1, 2])
def test_capacity_zero_drops_everything(k):
    layer, res, got = _edge(777, 128, 256, 4, k, 0)
    assert np.all(got == 0.0) and np.all(res["disp"]["drop"] == 1)


@pytest.mark.parametrize("k", [1, 2])
def test_capacity_at_least_T_keeps_everything(k):
    layer, res, got = _edge(1025, 128, 256, 4, k, 1025)
    assert not res["disp"]["drop"].any()


def test_single_expert_is_dense_ffn():
    layer, res, got = _edge(300, 128, 384, 1, 1, 300)
    assert np.all(res["routing"]["gate"] == 1.0)


def test_every_token_to_one_expert():
    bias = np.full(8, -20.0, np.float32)
    bias[3] = 0.0
    layer, res, got = _edge(2500, 128, 256, 8, 1, 400, router_bias=bias)
    assert res["disp"]["counts"][0, 3] == 2500 and res["disp"]["kept"][3] == 400
    assert np.all(got[400:] == 0.0) and np.all(np.abs(got[:400]).sum(1) > 0)


@pytest.mark.parametrize("T,C", [(2500, 400), (6000, 50)])
def test_dropped_rows_zeroed_over_stale_output(T, C):
    # top-1 bf16: the second GEMM writes only the kept tokens' rows, and the
    # dispatch zeroes the rows of dropped tokens.  The output starts as NaN
    # before each of two calls, and every dropped row must come back exactly 0
    # (most tokens are dropped here), the rest identical to the first call.
    bias = np.full(8, -20.0, np.float32)
    bias[3] = 0.0
    bias[5] = -0.5
    layer, res, got = _edge(T, 128, 256, 8, 1, C, router_bias=bias)
    drop = res["disp"]["drop"][:, 0].astype(bool)
    assert drop.sum() > T // 2
    x = to_device(inputs.make_layer(T=T, d_model=128, d_ff=256, n_experts=8, top_k=1, seed=3,
                                    router_bias=bias)["x"])
    for _ in range(2):
        layer.out.view(torch.int16).fill_(-1)   # bf16 0xFFFF: NaN
        nat.check(layer.forward(x))
        torch.cuda.synchronize()
        again = widen_out(layer.out)
        assert np.all(again[drop] == 0.0)
        np.testing.assert_array_equal(again, got)


def test_zero_router_ties_lowest_index():
    layer, res, got = _edge(333, 64, 128, 8, 2, 333, w_r_zero=True)
    assert np.all(res["routing"]["idx"][:, 0] == 0) and np.all(res["routing"]["idx"][:, 1] == 1)


def test_empty_experts_and_tiny_T():
    bias = np.zeros(16, np.float32)
    bias[8:] = -30.0
    _edge(200, 128, 256, 16, 2, 40, router_bias=bias)
    _edge(1, 128, 256, 16, 1, 1)
    _edge(3, 64, 64, 2, 2, 1, act="swiglu")


def test_empty_batch():
    T, d, dff, N, k = 0, 128, 256, 4, 2
    L = inputs.make_layer(T=0, d_model=d, d_ff=dff, n_experts=N, top_k=k, seed=1)
    layer, _ = run_layer(L, T, d, dff, N, k, 0, "bf16", "relu")
    assert layer.aux.item() == 0.0
    assert not layer.counts.any().item() and not layer.offsets.any().item()


def test_deterministic_bitwise():
    case = SMALL[1]
    T, d, dff, N, k, cf, act, dtype, biases = case
    L = _route_inputs(case, seed=9)
    C = nat.moe_capacity(T, N, k, cf)
    l1, x = run_layer(L, T, d, dff, N, k, C, dtype, act)
    a = to_host_bits(l1.out).copy()
    aux = l1.aux.item()
    nat.check(l1.forward(x))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host_bits(l1.out), a)
    assert l1.aux.item() == aux


def test_lookback_timeout_is_reported_and_context_survives():
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    assert nat.moe_read_device_status(ws) == nat.MOE_OK
    nat.check(nat.moe_test_lookback_timeout(ws, 20_000_000))   # 20 ms: the predecessor never publishes
    assert nat.moe_read_device_status(ws) == nat.MOE_ERR_TIMEOUT
    assert nat.moe_read_device_status(ws) == nat.MOE_OK          # cleared by the read
    _edge(100, 64, 64, 2, 1, 100)                                  # the context is still usable


# ------------------------------------------------------ full-size workloads ----

@pytest.mark.parametrize("name", ["tiny_f32", "switch_base", "top2", "skew", "mixtral"])
def test_workload_full_size(name):
    w = WORKLOADS[name]
    L = workload_inputs(name)
    C = nat.moe_capacity(w.T, w.n_experts, w.top_k, w.capacity_factor)
    layer, _ = run_layer(L, w.T, w.d_model, w.d_ff, w.n_experts, w.top_k, C, w.dtype, w.act, w.alpha)
    r = oracle.route(L["x"], L["w_r"], L["b_r"], w.top_k)
    dd = oracle.dispatch(r["idx"], w.n_experts, C)
    # sampled tokens (first/last/random/dropped) plus, for every expert, rows that
    # put a checked row in every m-tile of both expert GEMMs, including the last
    # row of every ragged tile (128-row slices; 256 for the costly Mixtral experts,
    # the CTA-pair tile height)
    tokens = None
    if w.T > 1024:
        tokens = np.union1d(sample_tokens(w.T, dd["drop"].astype(bool), n_random=24 if w.d_ff < 8192 else 8),
                            tile_cover_tokens(r["idx"], dd, 256 if w.d_ff >= 8192 else 128))
    res = oracle_layer_threads(L, w.top_k, C, w.act, w.dtype, w.alpha, tokens=tokens)
    compare_routing(layer, res)
    got = widen_out(layer.out)
    toks = res["tokens"]
    assert_close_out(got[toks], res["out_exact"], w.dtype)
    # every token with no kept assignment is exactly zero, at any size
    all_drop = dd["drop"].all(axis=1)
    assert np.all(got[all_drop] == 0.0)
    # router z-loss at full size, against the oracle's logits
    z = torch.empty(1, dtype=torch.float64, device="cuda")
    x = to_device(L["x"])
    nat.check(nat.moe_route_z(layer.cfg, x, layer.w["w_r"], layer.w["b_r"], layer.idx, layer.gate, None, None,
                              None, None, z, layer.ws))
    assert_rel(z.item(), oracle.z_loss(r["logits"]), REL_PROB, "z-loss")


def test_mixtral_literal_capacity():
    # the literal reading C = floor(T / N * cf) (no k factor) drops assignments even
    # under balanced routing; the path must still match the oracle under it
    w = WORKLOADS["mixtral"]
    L = workload_inputs("mixtral")
    C = nat.moe_capacity(w.T, w.n_experts, 1, w.capacity_factor)
    assert C == 2560
    layer, _ = run_layer(L, w.T, w.d_model, w.d_ff, w.n_experts, w.top_k, C, w.dtype, w.act, w.alpha)
    r = oracle.route(L["x"], L["w_r"], L["b_r"], w.top_k)
    dd = oracle.dispatch(r["idx"], w.n_experts, C)
    tokens = np.union1d(sample_tokens(w.T, dd["drop"].astype(bool), n_random=4), tile_cover_tokens(r["idx"], dd, 256))
    res = oracle_layer_threads(L, w.top_k, C, w.act, w.dtype, w.alpha, tokens=tokens)
    compare_routing(layer, res)
    assert_close_out(widen_out(layer.out)[res["tokens"]], res["out_exact"], w.dtype)


def test_single_cta_gemm_variant_in_subprocess():
    # the one-CTA (M=128) grouped GEMM, selected by MOE_B200_GEMM=single at
    # library load, must match the oracle as well
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "from test_gpu_parity import SMALL, test_forward_small_full_oracle\n"
        "for case in (SMALL[0], SMALL[1], SMALL[2], SMALL[4], SMALL[8]):\n"
        "    test_forward_small_full_oracle(case)\n"
        "print('single ok')\n" % (root, os.path.join(root, "tests")))
    env = dict(os.environ, MOE_B200_GEMM="single")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "single ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
