"""CPU oracle for the sparse MoE FFN layer forward -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The product path (the CUDA library and its binding) never does.

The arithmetic lives in ``moe_oracle.c`` (plain C, double accumulation,
single-threaded); this module only marshals numpy arrays into it.  Each function
names the passage of the pages it follows; the C source states the readings
taken where the pages are silent.

Parity status: every function here is pinned by tests/test_oracle_pins.py
against values the pages print, closed forms, special cases and brute force.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16 = 0, 1
RELU, SWIGLU = 0, 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        sz = ctypes.c_size_t
        lib.oracle_float_to_bf16_bits.argtypes = [ctypes.c_float]
        lib.oracle_float_to_bf16_bits.restype = ctypes.c_uint16
        lib.oracle_float_to_bf16_array.argtypes = [P, P, i64]
        lib.oracle_float_to_bf16_array.restype = None
        lib.oracle_bf16_round.argtypes = [ctypes.c_float]
        lib.oracle_bf16_round.restype = ctypes.c_float
        lib.oracle_router.argtypes = [i64, i32, i32, i32, P, i32, P, P, P, P, P, P]
        lib.oracle_router.restype = None
        lib.oracle_aux.argtypes = [i64, i32, i32, P, P, f64, P, P, P]
        lib.oracle_aux.restype = None
        lib.oracle_z_loss.argtypes = [i64, i32, P]
        lib.oracle_z_loss.restype = f64
        lib.oracle_capacity.argtypes = [i64, i32, i32, f64]
        lib.oracle_capacity.restype = i32
        lib.oracle_dispatch.argtypes = [i64, i32, i32, i32, P, P, P, P, P, P]
        lib.oracle_dispatch_ordered.argtypes = [i64, i32, i32, i32, P, P, P, P, P, P, P]
        lib.oracle_dispatch_ntlb.argtypes = [i64, i32, i32, P, P, P, P, P, P, P, P, P]
        lib.oracle_router_backward.argtypes = [i64, i32, i32, i32, P, i32, P, P, P, P, P, P, f64, P, P, P, P]
        lib.oracle_expert_backward.argtypes = [i64, i32, i32, i32, i32, i32, P, i32, P, P, P, P, P, P, i32,
                                               P, P, P, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_dispatch.restype = None
        lib.oracle_expert_ffn.argtypes = [i32, i32, i32, P, i32, sz, P, P, P, P, P, P, i32,
                                          sz, sz, sz, sz, P, P]
        lib.oracle_expert_ffn.restype = None
        lib.oracle_layer_tokens.argtypes = [i32, i32, i32, i32, P, i32, P, P, P, P, P, P, i32,
                                            P, P, P, i64, P, i32, P, P, P]
        lib.oracle_layer_tokens.restype = None
        lib.oracle_expert_rows.argtypes = [i32, i32, i32, P, i32, P, P, P, P, P, P, i32,
                                           i64, P, P, P, P]
        lib.oracle_expert_rows.restype = None
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _as_input(a):
    """Return (contiguous array, dtype code).  uint16 arrays are bf16 bit patterns."""
    if a is None:
        return None, F32
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, BF16
    if a.dtype != np.float32:
        raise TypeError(f"oracle inputs are float32 or bf16 bit patterns (uint16), got {a.dtype}")
    return a, F32


def bf16_bits(v):
    """fp32 -> bf16 bit pattern, round to nearest even (format definition)."""
    lib = _load()
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(v.shape, dtype=np.uint16)
    lib.oracle_float_to_bf16_array(_ptr(v), _ptr(out), v.size)
    return out


def bf16_round(v):
    """fp32 -> nearest bf16 value (ties to even), returned as fp32."""
    lib = _load()
    return np.float32(lib.oracle_bf16_round(float(v)))


def widen(a):
    """bf16 bit patterns (uint16) or fp32 -> fp64 values (exact)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def route(x, w_r, b_r=None, k=1):
    """Router of the MoE layer: fp32 logits, softmax, top-k, gate.

    Follows "From Switch Transformer to GLaM", sections "Dense Scaling vs MoE"
    (h = W_r x, softmax) and "Switch Transformer: making MoE simple" (top-1,
    y = p_{i*} E_{i*}), and CMU 10-423 Lecture 16 section 2.3 (top-k then
    softmax over the kept logits; ties to the lower index).
    Returns dict(logits, probs, idx, gate).
    """
    lib = _load()
    x, xd = _as_input(x)
    T, d = x.shape
    w_r = np.ascontiguousarray(w_r, dtype=np.float32)
    N = w_r.shape[0]
    assert w_r.shape == (N, d) and 1 <= k <= 2 and k <= N
    b = None if b_r is None else np.ascontiguousarray(b_r, dtype=np.float32)
    logits = np.empty((T, N), np.float32)
    probs = np.empty((T, N), np.float32)
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float32)
    lib.oracle_router(T, d, N, k, _ptr(x), xd, _ptr(w_r), _ptr(b), _ptr(logits), _ptr(probs),
                      _ptr(idx), _ptr(gate))
    return dict(logits=logits, probs=probs, idx=idx, gate=gate)


def z_loss(logits):
    """Router z-loss: the mean over tokens of (log sum_i exp h_i)^2 over the
    fp32 router logits (CMU 10-423 Lecture 16, section 4.2, "router z-loss";
    the page's formula is not legible, its experiment reports the router's
    logsumexp^2 -- this is that reading, unweighted)."""
    lib = _load()
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, N = logits.shape
    return float(lib.oracle_z_loss(T, N, _ptr(logits)))


def router_backward(x, w_r, probs, idx, gate, f, dgate, alpha=1e-2):
    """Router backward: gradients of sum dgate * gate + L_aux with respect to
    the router logits, W_r, b_r and x (gate path of "From Switch Transformer to
    GLaM"; load-balancing gradient through P_i with coefficient f_i, CMU 10-423
    Lecture 16 section 4.2).  Returns dict(dh [T,N], dw [N,d], db [N], dx [T,d])
    in fp64."""
    lib = _load()
    x, xd = _as_input(x)
    T, d = x.shape
    w_r = np.ascontiguousarray(w_r, dtype=np.float32)
    N = w_r.shape[0]
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    k = idx.shape[1]
    gate = np.ascontiguousarray(gate, dtype=np.float32)
    f = np.ascontiguousarray(f, dtype=np.float64)
    dgate = np.ascontiguousarray(dgate, dtype=np.float32)
    dh = np.empty((T, N), np.float64)
    dw = np.empty((N, d), np.float64)
    db = np.empty(N, np.float64)
    dx = np.empty((T, d), np.float64)
    lib.oracle_router_backward(T, d, N, k, _ptr(x), xd, _ptr(w_r), _ptr(probs), _ptr(idx), _ptr(gate), _ptr(f),
                               _ptr(dgate), float(alpha), _ptr(dh), _ptr(dw), _ptr(db), _ptr(dx))
    return dict(dh=dh, dw=dw, db=db, dx=dx)


def expert_backward(x, weights, idx, gate, drop, dout, act=RELU):
    """Expert-path backward of L = sum_t <dout_t, out_t>: dL/dgate, the expert
    part of dL/dx and the expert weight and bias gradients ("From Switch
    Transformer to GLaM" FFN; CMU 10-423 Lecture 16 section 2.3 SwiGLU).
    weights: dict(w1, b1, w3, b3, w2, b2) as for layer_tokens.  Returns a dict
    of fp64 arrays (dw3/db3 None for ReLU)."""
    lib = _load()
    x, xd = _as_input(x)
    T, d = x.shape
    w1, wd = _as_input(weights["w1"])
    N, d_ff, _ = w1.shape
    w2, _ = _as_input(weights["w2"])
    w3, _ = _as_input(weights.get("w3"))
    b1, _ = _as_input(weights.get("b1"))
    b3, _ = _as_input(weights.get("b3"))
    b2, _ = _as_input(weights.get("b2"))
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    k = idx.shape[1]
    gate = np.ascontiguousarray(gate, dtype=np.float32)
    drop = np.ascontiguousarray(drop, dtype=np.uint8)
    dout = np.ascontiguousarray(dout, dtype=np.float32)
    sw = act == SWIGLU
    out = dict(dgate=np.empty((T, k)), dx=np.empty((T, d)), dw1=np.empty((N, d_ff, d)), db1=np.empty((N, d_ff)),
               dw3=np.empty((N, d_ff, d)) if sw else None, db3=np.empty((N, d_ff)) if sw else None,
               dw2=np.empty((N, d, d_ff)), db2=np.empty((N, d)))
    scratch = np.empty(6 * d_ff, np.float64)
    lib.oracle_expert_backward(T, d, d_ff, N, k, act, _ptr(x), xd, _ptr(w1), _ptr(b1), _ptr(w3), _ptr(b3), _ptr(w2),
                               _ptr(b2), wd, _ptr(idx), _ptr(gate), _ptr(drop), _ptr(dout), _ptr(scratch),
                               _ptr(out["dgate"]), _ptr(out["dx"]), _ptr(out["dw1"]), _ptr(out["db1"]),
                               _ptr(out["dw3"]), _ptr(out["db3"]), _ptr(out["dw2"]), _ptr(out["db2"]))
    return out


def aux_loss(idx, probs, alpha=1e-2):
    """Load-balancing loss alpha N sum f_i P_i ("From Switch Transformer to
    GLaM", section "Load balancing").  Returns (f, P, aux) in fp64."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    T, N = probs.shape
    k = idx.shape[1]
    f = np.empty(N, np.float64)
    P = np.empty(N, np.float64)
    aux = np.empty(1, np.float64)
    lib.oracle_aux(T, N, k, _ptr(idx), _ptr(probs), float(alpha), _ptr(f), _ptr(P), _ptr(aux))
    return f, P, float(aux[0])


def capacity(T, N, k, cf):
    """Expert capacity floor(k T cf / N) (CMU 10-423 Lecture 16, exercise 3;
    "From Switch Transformer to GLaM", "Expert Capacity and Token Dropping")."""
    return int(_load().oracle_capacity(int(T), int(N), int(k), float(cf)))


def priority_order(gate):
    """Batch-priority claim order: tokens by descending priority score, ties to
    the lower token index.  CS25 Lecture 05 notes, section "from language MoE
    to Vision MoE": with a capacity factor below 1, priority routing first
    scores each token's importance and lets the high-priority tokens take the
    expert slots.  The score read here is the token's first-choice gate
    gate[t, 0] (the router's weight for its first choice), compared as fp32."""
    g0 = np.ascontiguousarray(np.asarray(gate, np.float32)[:, 0])
    T = g0.shape[0]
    return np.lexsort((np.arange(T), -g0.astype(np.float64))).astype(np.int64)


def dispatch(idx, N, C, priority=None):
    """Capacity-limited slot claim: rank-major, then token order (CS25 Lecture 05
    notes, capacity-aware dispatch; CMU 10-423 Lecture 16 section 6.1, GShard
    rule), or with priority=gate [T, k] the batch-priority order of
    priority_order(gate) (CS25 Lecture 05 notes, section "from language MoE to
    Vision MoE": priority routing).  Returns dict(pos, drop, counts[k,N], kept[N],
    offsets[N+1])."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    pos = np.empty((T, k), np.int32)
    drop = np.empty((T, k), np.uint8)
    counts = np.empty((k, N), np.int32)
    kept = np.empty(N, np.int32)
    offsets = np.empty(N + 1, np.int32)
    if priority is None:
        lib.oracle_dispatch(T, N, k, int(C), _ptr(idx), _ptr(pos), _ptr(drop), _ptr(counts),
                            _ptr(kept), _ptr(offsets))
    else:
        order = np.ascontiguousarray(priority_order(priority))
        lib.oracle_dispatch_ordered(T, N, k, int(C), _ptr(idx), _ptr(order), _ptr(pos), _ptr(drop),
                                    _ptr(counts), _ptr(kept), _ptr(offsets))
    return dict(pos=pos, drop=drop, counts=counts, kept=kept, offsets=offsets)


def dispatch_ntlb(probs, gate0, C):
    """No-Token-Left-Behind re-routing for top-1 (CS25 Lecture 05 notes, "No
    Token Left Behind": a token whose expert is full goes on to its next
    choices until it gets a slot).  Stages in token order; see the C source for
    the reading.  Returns dict(expert, gate, pos, drop, counts[N], kept[N],
    offsets[N+1])."""
    lib = _load()
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    T, N = probs.shape
    gate0 = np.ascontiguousarray(np.asarray(gate0, np.float32).reshape(T))
    expert = np.empty(T, np.int32)
    gate = np.empty(T, np.float32)
    pos = np.empty(T, np.int32)
    drop = np.empty(T, np.uint8)
    counts = np.empty(N, np.int32)
    kept = np.empty(N, np.int32)
    offsets = np.empty(N + 1, np.int32)
    lib.oracle_dispatch_ntlb(T, N, int(C), _ptr(probs), _ptr(gate0), _ptr(expert), _ptr(gate), _ptr(pos),
                             _ptr(drop), _ptr(counts), _ptr(kept), _ptr(offsets))
    return dict(expert=expert, gate=gate, pos=pos, drop=drop, counts=counts, kept=kept, offsets=offsets)


def expert_ffn(x_row, w1, b1, w2, b2, act=RELU, w3=None, b3=None):
    """One expert on one token, in fp64 ("From Switch Transformer to GLaM",
    FFN(x) = W2 s(W1 x); CMU 10-423 Lecture 16 section 2.3, SwiGLU expert).
    w1, w3: [d_ff, d]; w2: [d, d_ff]; biases optional."""
    lib = _load()
    x_row, xd = _as_input(np.asarray(x_row).reshape(1, -1))
    d = x_row.shape[1]
    w1, wd = _as_input(w1)
    d_ff = w1.shape[0]
    w2, wd2 = _as_input(w2)
    assert wd == wd2 and w1.shape == (d_ff, d) and w2.shape == (d, d_ff)
    w3, _ = _as_input(w3)
    b1, _ = _as_input(b1)
    b2, _ = _as_input(b2)
    b3, _ = _as_input(b3)
    if act == SWIGLU:
        assert w3 is not None
    scratch = np.empty(d_ff, np.float64)
    y = np.empty(d, np.float64)
    lib.oracle_expert_ffn(d, d_ff, act, _ptr(x_row), xd, 0, _ptr(w1), _ptr(b1), _ptr(w3), _ptr(b3),
                          _ptr(w2), _ptr(b2), wd, 0, 0, 0, 0, _ptr(scratch), _ptr(y))
    return y


def layer_tokens(x, weights, routing, disp, tokens, act=RELU, out_dtype=F32):
    """Layer output for selected tokens: out_t = sum over kept r of
    g_{t,r} E_{idx}(x_t), zero when every assignment of t is dropped ("From
    Switch Transformer to GLaM", top-1/top-2 output and token dropping).
    weights: dict(w1, b1, w3, b3, w2, b2) with w1/w3 [N, d_ff, d], w2 [N, d, d_ff].
    Returns (exact fp64 [n, d], rounded fp32 [n, d])."""
    lib = _load()
    x, xd = _as_input(x)
    T, d = x.shape
    w1, wd = _as_input(weights["w1"])
    N, d_ff, _ = w1.shape
    w2, _ = _as_input(weights["w2"])
    w3, _ = _as_input(weights.get("w3"))
    b1, _ = _as_input(weights.get("b1"))
    b3, _ = _as_input(weights.get("b3"))
    b2, _ = _as_input(weights.get("b2"))
    idx = np.ascontiguousarray(routing["idx"], dtype=np.int32)
    gate = np.ascontiguousarray(routing["gate"], dtype=np.float32)
    drop = np.ascontiguousarray(disp["drop"], dtype=np.uint8)
    k = idx.shape[1]
    tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64).reshape(-1))
    n = tokens.size
    scratch = np.empty(d_ff + d, np.float64)
    out_exact = np.empty((n, d), np.float64)
    out_rounded = np.empty((n, d), np.float32)
    lib.oracle_layer_tokens(d, d_ff, k, act, _ptr(x), xd, _ptr(w1), _ptr(b1), _ptr(w3), _ptr(b3),
                            _ptr(w2), _ptr(b2), wd, _ptr(idx), _ptr(gate), _ptr(drop), n,
                            _ptr(tokens), out_dtype, _ptr(scratch), _ptr(out_exact),
                            _ptr(out_rounded))
    return out_exact, out_rounded


def expert_rows(x, weights, rows_token, rows_expert, act=RELU):
    """Un-gated expert outputs E_e(x_t) for the given (token, expert) rows, fp64."""
    lib = _load()
    x, xd = _as_input(x)
    T, d = x.shape
    w1, wd = _as_input(weights["w1"])
    N, d_ff, _ = w1.shape
    w2, _ = _as_input(weights["w2"])
    w3, _ = _as_input(weights.get("w3"))
    b1, _ = _as_input(weights.get("b1"))
    b3, _ = _as_input(weights.get("b3"))
    b2, _ = _as_input(weights.get("b2"))
    rt = np.ascontiguousarray(np.asarray(rows_token, dtype=np.int64).reshape(-1))
    re = np.ascontiguousarray(np.asarray(rows_expert, dtype=np.int32).reshape(-1))
    scratch = np.empty(d_ff, np.float64)
    ye = np.empty((rt.size, d), np.float64)
    lib.oracle_expert_rows(d, d_ff, act, _ptr(x), xd, _ptr(w1), _ptr(b1), _ptr(w3), _ptr(b3),
                           _ptr(w2), _ptr(b2), wd, rt.size, _ptr(rt), _ptr(re), _ptr(scratch),
                           _ptr(ye))
    return ye


def forward(x, w_r, b_r, weights, k, C, act=RELU, alpha=1e-2, out_dtype=F32, tokens=None, priority=False,
            ntlb=False):
    """The whole layer, step by step: route, aux loss, slot claim (token order,
    batch priority, or No-Token-Left-Behind re-routing for top-1), experts,
    combine.  tokens=None evaluates every token.  Returns a dict with every
    intermediate and the outputs for the evaluated tokens; with ntlb the
    experts and gates used are in disp["expert"] / disp["gate"]."""
    routing = route(x, w_r, b_r, k)
    f, P, aux = aux_loss(routing["idx"], routing["probs"], alpha)
    N = np.asarray(w_r).shape[0]
    if ntlb:
        assert k == 1
        disp = dispatch_ntlb(routing["probs"], routing["gate"][:, 0], C)
        used = dict(idx=disp["expert"][:, None], gate=disp["gate"][:, None])
        T = np.asarray(x).shape[0]
        if tokens is None:
            tokens = np.arange(T, dtype=np.int64)
        out_exact, out_rounded = layer_tokens(x, weights, used, dict(drop=disp["drop"][:, None]), tokens, act,
                                              out_dtype)
        return dict(routing=routing, f=f, P=P, aux=aux, disp=disp, tokens=np.asarray(tokens),
                    out_exact=out_exact, out=out_rounded)
    disp = dispatch(routing["idx"], N, C, priority=routing["gate"] if priority else None)
    T = np.asarray(x).shape[0]
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    out_exact, out_rounded = layer_tokens(x, weights, routing, disp, tokens, act, out_dtype)
    return dict(routing=routing, f=f, P=P, aux=aux, disp=disp, tokens=np.asarray(tokens),
                out_exact=out_exact, out=out_rounded)
