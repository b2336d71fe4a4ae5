"""Seeded synthetic inputs for the MoE layer (shared by the tests, the smoke
check and the benchmark; holds none of the layer's own arithmetic).

Recipe (the pages' stability settings, "Training Stability, Results &
Limitations", section 2.2, and "From Switch Transformer to GLaM"):
  * x ~ N(0, 1) per element, then per-row LayerNorm (no affine, eps 1e-5) or
    RMSNorm (eps 1e-6), then cast to the activation dtype (bf16: round to
    nearest even);
  * every weight matrix from a normal truncated at 2 sigma (out-of-range draws
    are redrawn), sigma = sqrt(0.1 / fan_in); fan_in is d_model for W_r, W1,
    W3 and d_ff for W2; optional biases use the same law and fan-in; each
    expert's matrix comes from its own child seed stream;
  * the router W_r stays fp32; expert weights take the activation dtype;
  * skewed routing: router bias b_r[i] = 3 ln(pi_i), pi_i proportional to
    (i + 1)^-s over the experts;
  * gap guard: any token whose top-1/top-2 router logit gap (and, for top-2,
    the 2nd/3rd gap) is below 1e-4 on the final logits is redrawn, so the
    discrete routing is unique.
bf16 tensors are returned as uint16 bit patterns.
"""
import concurrent.futures
import os

import numpy as np

GAP = 1e-4


def _threads():
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1))


def _bf16_bits(a32):
    """fp32 -> bf16 bit patterns, round to nearest even (input casting only)."""
    u = np.ascontiguousarray(a32, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _trunc_normal(rng, shape, sigma):
    out = rng.standard_normal(shape, dtype=np.float32)
    bad = np.abs(out) > 2.0
    while bad.any():
        out[bad] = rng.standard_normal(int(bad.sum()), dtype=np.float32)
        bad = np.abs(out) > 2.0
    out *= np.float32(sigma)
    return out


def _normalise(rows, norm):
    r = rows.astype(np.float64)
    if norm == "layernorm":
        mu = r.mean(axis=1, keepdims=True)
        var = ((r - mu) ** 2).mean(axis=1, keepdims=True)
        r = (r - mu) / np.sqrt(var + 1e-5)
    elif norm == "rmsnorm":
        r = r / np.sqrt((r * r).mean(axis=1, keepdims=True) + 1e-6)
    else:
        raise ValueError(norm)
    return r.astype(np.float32)


def _draw_x(rng, n, d, norm, dtype):
    x32 = _normalise(rng.standard_normal((n, d), dtype=np.float32), norm)
    if dtype == "bf16":
        bits = _bf16_bits(x32)
        return bits, bf16_to_f32(bits)
    return x32, x32


def zipf_router_bias(N, s):
    pop = (np.arange(N, dtype=np.float64) + 1.0) ** (-s)
    pop /= pop.sum()
    return (3.0 * np.log(pop)).astype(np.float32)


def _small_gap(x_val, w_r, b_r, k):
    h = x_val.astype(np.float64) @ w_r.astype(np.float64).T
    if b_r is not None:
        h += b_r.astype(np.float64)[None, :]
    if h.shape[1] < 2:
        return np.zeros(h.shape[0], dtype=bool)
    top = -np.sort(-h, axis=1)
    bad = (top[:, 0] - top[:, 1]) < GAP
    if k == 2 and h.shape[1] >= 3:
        bad |= (top[:, 1] - top[:, 2]) < GAP
    return bad


def make_layer(T, d_model, d_ff, n_experts, top_k=1, act="relu", dtype="bf16",
               norm="layernorm", biases=False, zipf_exponent=None, seed=0,
               router_bias=None, gap_guard=True, x_seed=None, **_ignored):
    """Build one layer's inputs and weights.

    Returns a dict of numpy arrays: x [T, d] (uint16 bf16 bits or fp32), w_r
    [N, d] fp32, b_r [N] fp32 or None, w1 [N, d_ff, d], w3 (SwiGLU) or None,
    w2 [N, d, d_ff], b1 [N, d_ff] / b3 / b2 [N, d] or None.  x_seed (optional)
    draws x from its own seed while the weights still come from `seed` (the
    shards of one routing group share the weights).
    """
    ss = np.random.SeedSequence(seed)
    s_x, s_r, s_1, s_3, s_2, s_b = ss.spawn(6)
    if x_seed is not None:
        s_x = np.random.SeedSequence(x_seed).spawn(1)[0]
    N, d = n_experts, d_model
    rng_r = np.random.default_rng(s_r)
    w_r = _trunc_normal(rng_r, (N, d), np.sqrt(0.1 / d))
    if router_bias is not None:
        b_r = np.asarray(router_bias, dtype=np.float32)
    elif zipf_exponent is not None:
        b_r = zipf_router_bias(N, zipf_exponent)
    else:
        b_r = None

    rng_x = np.random.default_rng(s_x)
    x_store, x_val = _draw_x(rng_x, T, d, norm, dtype)
    if gap_guard and T > 0:
        for _ in range(1000):
            bad = np.nonzero(_small_gap(x_val, w_r, b_r, top_k))[0]
            if bad.size == 0:
                break
            new_store, new_val = _draw_x(rng_x, bad.size, d, norm, dtype)
            x_store[bad] = new_store
            x_val[bad] = new_val
        else:
            raise RuntimeError("gap guard did not converge")

    def weight(seed_seq, shape, fan_in):
        # one child stream per expert, so the experts can be drawn on several
        # host threads (numpy's generators release the GIL while filling)
        sigma = np.sqrt(0.1 / fan_in)
        out = np.empty(shape, dtype=np.uint16 if dtype == "bf16" else np.float32)

        def draw(e, ss):
            w = _trunc_normal(np.random.default_rng(ss), shape[1:], sigma)
            out[e] = _bf16_bits(w) if dtype == "bf16" else w

        children = seed_seq.spawn(shape[0])
        if out.nbytes < (64 << 20):
            for e, ss in enumerate(children):
                draw(e, ss)
        else:
            with concurrent.futures.ThreadPoolExecutor(max_workers=min(shape[0], _threads())) as ex:
                list(ex.map(lambda a: draw(*a), enumerate(children)))
        return out

    w1 = weight(s_1, (N, d_ff, d), d)
    w3 = weight(s_3, (N, d_ff, d), d) if act == "swiglu" else None
    w2 = weight(s_2, (N, d, d_ff), d_ff)
    b1 = b3 = b2 = None
    if biases:
        b1s, b3s, b2s = s_b.spawn(3)
        b1 = weight(b1s, (N, d_ff), d)
        b3 = weight(b3s, (N, d_ff), d) if act == "swiglu" else None
        b2 = weight(b2s, (N, d), d_ff)
    return dict(x=x_store, w_r=w_r, b_r=b_r, w1=w1, w3=w3, w2=w2, b1=b1, b3=b3, b2=b2)


def make_workload(w, x_seed=None, **overrides):
    """Inputs for a configs.Workload (fields may be overridden, e.g. T=...)."""
    w = w.scaled(**overrides) if overrides else w
    return make_layer(T=w.T, d_model=w.d_model, d_ff=w.d_ff, n_experts=w.n_experts,
                      top_k=w.top_k, act=w.act, dtype=w.dtype, norm=w.norm, biases=w.biases,
                      zipf_exponent=w.zipf_exponent, seed=w.seed, x_seed=x_seed)
