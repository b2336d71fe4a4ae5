/*
 * CPU oracle for the forward pass of one sparse Mixture-of-Experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously correct
 * statement of what the layer computes.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * table or helper with the CUDA library, and it never reads a value that the
 * CUDA library produced.
 *
 * Arithmetic: every sum is accumulated in double in ascending index order; the
 * only roundings are the ones the definitions below state.  Inputs arrive as
 * fp32 values or as raw bf16 bit patterns; a bf16 value is widened to fp32 and
 * then to double exactly.
 *
 * Sources (page title, section):
 *  - "From Switch Transformer to GLaM" (blog.euler0525.cn), sections
 *    "Dense Scaling vs MoE" (FFN(x) = W2 s(W1 x); router h(x) = W_r x; softmax
 *    p_i), "Switch Transformer: making MoE simple" (top-1 i* = argmax p,
 *    y = p_{i*} E_{i*}(x)), "Load balancing" (f_i, P_i, L_aux = alpha N sum f_i
 *    P_i, alpha = 1e-2), "Expert Capacity and Token Dropping" (C = T/N x cf;
 *    an overflowing token skips the expert FFN and only the residual carries
 *    it), "Why GLaM returns to top-2" (y = w1 E_{i1} + w2 E_{i2}).
 *  - CMU 10-423 Lecture 16 "Mixture of Experts", section 2.3 (sparse gating
 *    G(x) = softmax(topk(x W_g, k)), non-top-k entries set to -inf; the
 *    Mixtral SwiGLU expert; a zero router picks the lowest indices on ties),
 *    section 6.1 (capacity with the GShard rule: all tokens' first choices are
 *    placed before any second choice), exercise 3 (C = cf k T / N = 320).
 *  - CS25 Lecture 05 notes "Scaling Transformers through Sparsity", section
 *    "Static compilation meets dynamic routing" (capacity-aware dispatch:
 *    tokens claim slots in token order, a full expert skips the token).
 *  - "Training Stability, Results & Limitations" (nano-ai.tech), section 2.1
 *    Selective Precision (router in float32; bf16 rounding example).
 *
 * Readings taken where the pages are silent or garbled:
 *  - top-k ties go to the lower expert index; the ranking uses the fp32 logits;
 *  - C = floor(k T cf / N), computed exactly from the double cf;
 *  - slot claim is rank-major (every rank-0 choice before any rank-1 choice),
 *    then token order;
 *  - gates are fixed before capacity: a surviving assignment keeps its gate;
 *  - a token with no kept assignment gets a zero layer output;
 *  - f_i counts the pre-capacity top-1 choice; P_i averages the full softmax;
 *  - Swish uses beta = 1: silu(z) = z / (1 + exp(-z));
 *  - biases are optional and are added inside the expert, before gating.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

#define ORACLE_RELU 0
#define ORACLE_SWIGLU 1

/* ---- bf16 <-> fp32, written from the format's definition ----------------
 * A bf16 value is the upper 16 bits of an IEEE-754 binary32 value.
 * Widening appends 16 zero bits (exact).  Narrowing rounds to nearest, ties to
 * even, on the 16 discarded bits; NaN stays NaN (quiet). */
static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

uint16_t oracle_float_to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u) {
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    }
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) {
        upper += 1u; /* carries into the exponent correctly, up to infinity */
    }
    return (uint16_t)upper;
}

void oracle_float_to_bf16_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_float_to_bf16_bits(in[i]);
}

float oracle_bf16_round(float f) {
    return bf16_bits_to_float(oracle_float_to_bf16_bits(f));
}

/* element i of an array that is fp32 or raw bf16, widened to double */
static double load_elem(const void* base, int dtype, size_t i) {
    if (dtype == ORACLE_BF16) {
        return (double)bf16_bits_to_float(((const uint16_t*)base)[i]);
    }
    return (double)((const float*)base)[i];
}

/* ---- Router: logits, softmax, top-k, gate --------------------------------
 * h_{t,i} = sum_j x_{t,j} W_r[i,j] (+ b_r[i]) in double, ascending j, then
 * rounded once to fp32 (the router is an fp32 computation).
 * p_{t,i} = exp(h_i - m) / sum_j exp(h_j - m), m = max_j h_j, in double,
 * stored as fp32 (the shift by m leaves the softmax value unchanged).
 * top-1: the largest h; on equal h the lower index.  top-2: the largest h
 * among the other experts, same tie rule.
 * gate, k = 1: p_{i*}.  k = 2: softmax over the two kept logits,
 * g_r = exp(h_{i_r} - h_{i_1}) / (1 + exp(h_{i_2} - h_{i_1})).
 *
 * x: [T, d] (dtype x_dtype); w_r: [N, d] fp32; b_r: [N] fp32 or NULL.
 * Outputs: logits [T, N] fp32 (nullable), probs [T, N] fp32 (nullable),
 * idx [T, k] int32, gate [T, k] fp32. */
void oracle_router(int64_t T, int32_t d, int32_t N, int32_t k,
                   const void* x, int32_t x_dtype, const float* w_r, const float* b_r,
                   float* logits, float* probs, int32_t* idx, float* gate) {
    float h[1024];
    double e[1024];
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t i = 0; i < N; ++i) {
            double acc = 0.0;
            for (int32_t j = 0; j < d; ++j) {
                acc += load_elem(x, x_dtype, (size_t)t * d + j) * (double)w_r[(size_t)i * d + j];
            }
            if (b_r) acc += (double)b_r[i];
            h[i] = (float)acc;
        }
        double m = (double)h[0];
        for (int32_t i = 1; i < N; ++i) {
            if ((double)h[i] > m) m = (double)h[i];
        }
        double s = 0.0;
        for (int32_t i = 0; i < N; ++i) {
            e[i] = exp((double)h[i] - m);
            s += e[i];
        }
        for (int32_t i = 0; i < N; ++i) {
            if (logits) logits[(size_t)t * N + i] = h[i];
            if (probs) probs[(size_t)t * N + i] = (float)(e[i] / s);
        }
        int32_t i1 = 0;
        for (int32_t i = 1; i < N; ++i) {
            if (h[i] > h[i1]) i1 = i; /* strict: the lower index keeps a tie */
        }
        if (k == 1) {
            idx[t] = i1;
            gate[t] = (float)(e[i1] / s);
        } else {
            int32_t i2 = (i1 == 0) ? 1 : 0;
            for (int32_t i = 0; i < N; ++i) {
                if (i == i1) continue;
                if (h[i] > h[i2]) i2 = i;
            }
            double r = exp((double)h[i2] - (double)h[i1]);
            idx[t * 2 + 0] = i1;
            idx[t * 2 + 1] = i2;
            gate[t * 2 + 0] = (float)(1.0 / (1.0 + r));
            gate[t * 2 + 1] = (float)(r / (1.0 + r));
        }
    }
}

/* ---- Router z-loss --------------------------------------------------------
 * CMU 10-423 Lecture 16, section 4.2 ("router z-loss", Zoph et al. 2022): a
 * penalty on large router logits; the page's formula is not legible, and its
 * experiment reports the router's "logsumexp^2".  Reading taken:
 *   z = (1/T) sum_t ( log sum_i exp(h_{t,i}) )^2
 * over the fp32 router logits h (the values oracle_router writes), without the
 * weight (0.001 in OLMoE), which the caller applies.  log-sum-exp is taken as
 * m + log sum_i exp(h_i - m), m = max_i h_i, in double.  T = 0 gives 0. */
double oracle_z_loss(int64_t T, int32_t N, const float* logits) {
    if (T <= 0) return 0.0;
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        const float* h = logits + (size_t)t * N;
        double m = (double)h[0];
        for (int32_t i = 1; i < N; ++i) {
            if ((double)h[i] > m) m = (double)h[i];
        }
        double s = 0.0;
        for (int32_t i = 0; i < N; ++i) s += exp((double)h[i] - m);
        const double lse = m + log(s);
        acc += lse * lse;
    }
    return acc / (double)T;
}

/* ---- Load-balancing loss -------------------------------------------------
 * f_i = #{t : top-1 choice of t is i} / T   (pre-capacity, argmax indicator)
 * P_i = sum_t p_{t,i} / T
 * aux = alpha * N * sum_i f_i P_i
 * idx: [T, k]; its column 0 is the top-1 choice.  T = 0 gives all zeros. */
void oracle_aux(int64_t T, int32_t N, int32_t k, const int32_t* idx, const float* probs,
                double alpha, double* f, double* P, double* aux) {
    for (int32_t i = 0; i < N; ++i) {
        f[i] = 0.0;
        P[i] = 0.0;
    }
    *aux = 0.0;
    if (T <= 0) return;
    for (int64_t t = 0; t < T; ++t) {
        f[idx[t * k]] += 1.0;
        for (int32_t i = 0; i < N; ++i) P[i] += (double)probs[(size_t)t * N + i];
    }
    double s = 0.0;
    for (int32_t i = 0; i < N; ++i) {
        f[i] /= (double)T;
        P[i] /= (double)T;
        s += f[i] * P[i];
    }
    *aux = alpha * (double)N * s;
}

/* ---- Router backward -------------------------------------------------------
 * Gradient of L = sum_{t,r} dgate[t,r] g_{t,r}(h) + L_aux(h) with respect to the
 * router logits h, the router weights and bias, and the router's input x.
 *  - gate path ("From Switch Transformer to GLaM": y = p_{i*} E_{i*}(x) for
 *    top-1; y = w1 E_{i1} + w2 E_{i2} with w the softmax over the two kept
 *    logits for top-2; the expert choice itself has no gradient):
 *      top-1: g = p_{i*}, dg/dh_j = p_{i*} (delta_{j i*} - p_j);
 *      top-2: g1 = 1 / (1 + e^{h2 - h1}), g2 = 1 - g1; dg1/dh1 = -dg1/dh2 =
 *             g1 g2, and g2 the opposite.
 *  - load-balancing loss (CMU 10-423 Lecture 16, section 4.2: f_i is counted
 *    and carries no gradient; the gradient flows through P_i with coefficient
 *    f_i): dL_aux/dp_{t,i} = alpha N f_i / T, then through the softmax:
 *    dh_{t,j} = p_{t,j} (a_j - sum_i p_{t,i} a_i), a_i = alpha N f_i / T.
 *  - dW_r[i, :] = sum_t dh_{t,i} x_t, db_r[i] = sum_t dh_{t,i},
 *    dx_t = sum_i dh_{t,i} W_r[i, :]  (h = W_r x + b_r).
 * probs [T, N] and gate [T, k] are the forward's fp32 values; f [N] double.
 * Outputs in double: dh [T, N], dw [N, d], db [N], dx [T, d]. */
void oracle_router_backward(int64_t T, int32_t d, int32_t N, int32_t k,
                            const void* x, int32_t x_dtype, const float* w_r,
                            const float* probs, const int32_t* idx, const float* gate,
                            const double* f, const float* dgate, double alpha,
                            double* dh, double* dw, double* db, double* dx) {
    double a[1024];
    for (int32_t i = 0; i < N; ++i) a[i] = T > 0 ? alpha * (double)N * f[i] / (double)T : 0.0;
    for (int32_t i = 0; i < N; ++i) {
        db[i] = 0.0;
        for (int32_t j = 0; j < d; ++j) dw[(size_t)i * d + j] = 0.0;
    }
    for (int64_t t = 0; t < T; ++t) {
        const float* p = probs + (size_t)t * N;
        double* g = dh + (size_t)t * N;
        double spa = 0.0;
        for (int32_t i = 0; i < N; ++i) spa += (double)p[i] * a[i];
        for (int32_t j = 0; j < N; ++j) g[j] = (double)p[j] * (a[j] - spa);
        if (k == 1) {
            const int32_t is = idx[t];
            const double gs = (double)gate[t], dg = (double)dgate[t];
            for (int32_t j = 0; j < N; ++j) g[j] += dg * gs * ((j == is ? 1.0 : 0.0) - (double)p[j]);
        } else {
            const int32_t i1 = idx[t * 2], i2 = idx[t * 2 + 1];
            const double g1 = (double)gate[t * 2], g2 = (double)gate[t * 2 + 1];
            const double c = (double)dgate[t * 2] - (double)dgate[t * 2 + 1];
            g[i1] += c * g1 * g2;
            g[i2] -= c * g1 * g2;
        }
        for (int32_t i = 0; i < N; ++i) {
            db[i] += g[i];
            for (int32_t j = 0; j < d; ++j) dw[(size_t)i * d + j] += g[i] * load_elem(x, x_dtype, (size_t)t * d + j);
        }
        for (int32_t j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int32_t i = 0; i < N; ++i) acc += g[i] * (double)w_r[(size_t)i * d + j];
            dx[(size_t)t * d + j] = acc;
        }
    }
}

/* ---- Expert backward -------------------------------------------------------
 * Gradients of L = sum_t <dout_t, out_t> through the kept assignments of the
 * layer: out_t = sum_{kept r} g_{t,r} E_{e}(x_t) ("From Switch Transformer to
 * GLaM": FFN(x) = W2 s(W1 x); CMU 10-423 Lecture 16, section 2.3: the SwiGLU
 * expert silu(W1 x) * (W3 x)).  Per kept (t, r) with expert e and gate g:
 *   u = W1 x + b1, (v = W3 x + b3), a = relu(u) | silu(u) v, y = W2 a + b2;
 *   dgate[t,r] = <dout_t, y>;  dy = g dout_t;
 *   dW2[e] += dy a^T, db2[e] += dy, da = W2^T dy;
 *   ReLU:   du = da (u > 0);
 *   SwiGLU: du = da v silu'(u), dv = da silu(u), silu'(u) = s(u)(1 + u(1 - s(u)));
 *   dW1[e] += du x^T, db1[e] += du, (dW3[e] += dv x^T, db3[e] += dv);
 *   dx_t += W1^T du (+ W3^T dv).
 * Dropped assignments contribute nothing (dgate 0).  Weights as in
 * oracle_expert_ffn; outputs in double, zero-initialised here: dgate [T,k],
 * dx [T,d], dw1/dw3 [N,d_ff,d], db1/db3 [N,d_ff], dw2 [N,d,d_ff], db2 [N,d]
 * (dw3/db3 only for SwiGLU; they may be NULL otherwise). */
void oracle_expert_backward(int64_t T, int32_t d, int32_t d_ff, int32_t N, int32_t k, int32_t act,
                            const void* x, int32_t x_dtype,
                            const void* w1, const void* b1, const void* w3, const void* b3,
                            const void* w2, const void* b2, int32_t w_dtype,
                            const int32_t* idx, const float* gate, const uint8_t* drop, const float* dout,
                            double* scratch, double* dgate, double* dx, double* dw1, double* db1,
                            double* dw3, double* db3, double* dw2, double* db2) {
    double* u = scratch;
    double* v = u + d_ff;
    double* a = v + d_ff;
    double* da = a + d_ff;
    double* du = da + d_ff;
    double* dv = du + d_ff;
    const int swiglu = act == ORACLE_SWIGLU;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < d; ++j) dx[(size_t)t * d + j] = 0.0;
    for (size_t i = 0; i < (size_t)N * d_ff * d; ++i) {
        dw1[i] = 0.0;
        dw2[i] = 0.0;
        if (swiglu) dw3[i] = 0.0;
    }
    for (size_t i = 0; i < (size_t)N * d_ff; ++i) {
        db1[i] = 0.0;
        if (swiglu) db3[i] = 0.0;
    }
    for (size_t i = 0; i < (size_t)N * d; ++i) db2[i] = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t r = 0; r < k; ++r) {
            dgate[t * k + r] = 0.0;
            if (drop[t * k + r]) continue;
            const int32_t e = idx[t * k + r];
            const double g = (double)gate[t * k + r];
            const size_t o1 = (size_t)e * d_ff * d, ob1 = (size_t)e * d_ff, o2 = (size_t)e * d * d_ff,
                         ob2 = (size_t)e * d;
            for (int32_t j = 0; j < d_ff; ++j) {
                double su = 0.0, sv = 0.0;
                for (int32_t i = 0; i < d; ++i) {
                    const double xi = load_elem(x, x_dtype, (size_t)t * d + i);
                    su += load_elem(w1, w_dtype, o1 + (size_t)j * d + i) * xi;
                    if (swiglu) sv += load_elem(w3, w_dtype, o1 + (size_t)j * d + i) * xi;
                }
                if (b1) su += load_elem(b1, w_dtype, ob1 + j);
                if (swiglu && b3) sv += load_elem(b3, w_dtype, ob1 + j);
                u[j] = su;
                v[j] = sv;
                a[j] = swiglu ? su / (1.0 + exp(-su)) * sv : (su > 0.0 ? su : 0.0);
            }
            double dg = 0.0;
            for (int32_t n = 0; n < d; ++n) {
                double y = 0.0;
                for (int32_t j = 0; j < d_ff; ++j) y += load_elem(w2, w_dtype, o2 + (size_t)n * d_ff + j) * a[j];
                if (b2) y += load_elem(b2, w_dtype, ob2 + n);
                dg += (double)dout[(size_t)t * d + n] * y;
            }
            dgate[t * k + r] = dg;
            for (int32_t j = 0; j < d_ff; ++j) da[j] = 0.0;
            for (int32_t n = 0; n < d; ++n) {
                const double dy = g * (double)dout[(size_t)t * d + n];
                db2[ob2 + n] += dy;
                for (int32_t j = 0; j < d_ff; ++j) {
                    dw2[o2 + (size_t)n * d_ff + j] += dy * a[j];
                    da[j] += load_elem(w2, w_dtype, o2 + (size_t)n * d_ff + j) * dy;
                }
            }
            for (int32_t j = 0; j < d_ff; ++j) {
                if (swiglu) {
                    const double sg = 1.0 / (1.0 + exp(-u[j]));
                    du[j] = da[j] * v[j] * sg * (1.0 + u[j] * (1.0 - sg));
                    dv[j] = da[j] * u[j] * sg;
                } else {
                    du[j] = u[j] > 0.0 ? da[j] : 0.0;
                    dv[j] = 0.0;
                }
                db1[ob1 + j] += du[j];
                if (swiglu) db3[ob1 + j] += dv[j];
                for (int32_t i = 0; i < d; ++i) {
                    const double xi = load_elem(x, x_dtype, (size_t)t * d + i);
                    dw1[o1 + (size_t)j * d + i] += du[j] * xi;
                    dx[(size_t)t * d + i] += load_elem(w1, w_dtype, o1 + (size_t)j * d + i) * du[j];
                    if (swiglu) {
                        dw3[o1 + (size_t)j * d + i] += dv[j] * xi;
                        dx[(size_t)t * d + i] += load_elem(w3, w_dtype, o1 + (size_t)j * d + i) * dv[j];
                    }
                }
            }
        }
    }
}

/* ---- Capacity --------------------------------------------------------------
 * C = floor(k * T * cf / N), exact.  cf is a binary double m * 2^e with m an
 * odd-or-zero 53-bit integer, so k T cf / N = k T m / (N 2^-e) is a rational
 * whose floor is taken with 128-bit integers.  Returns -1 when the inputs are
 * out of range (T < 0, N < 1, k < 1, cf < 0 or not finite, result > 2^31-1). */
int32_t oracle_capacity(int64_t T, int32_t N, int32_t k, double cf) {
    if (T < 0 || N < 1 || k < 1 || !(cf >= 0.0) || isinf(cf)) return -1;
    if (cf == 0.0 || T == 0) return 0;
    int ex;
    double fr = frexp(cf, &ex);           /* cf = fr * 2^ex, 0.5 <= fr < 1 */
    int64_t m = (int64_t)ldexp(fr, 53);   /* exact: fr has 53 significant bits */
    ex -= 53;                             /* cf = m * 2^ex */
    while (m % 2 == 0 && ex < 0) {
        m /= 2;
        ex += 1;
    }
    __int128 num = (__int128)k * (__int128)T * (__int128)m;
    __int128 den = (__int128)N;
    if (ex >= 0) {
        if (ex > 60) return -1;
        num <<= ex;
    } else {
        if (-ex > 100) return 0;
        den <<= -ex;
    }
    __int128 q = num / den;
    if (q > (__int128)2147483647) return -1;
    return (int32_t)q;
}

/* ---- Capacity-limited slot claim -------------------------------------------
 * For r = 0..k-1, for the tokens in claim order: e = idx[t, r]; the assignment
 * takes claim number pos[t, r] = (claims on e so far); it is kept iff pos < C.
 * The claim order is token order (CS25 Lecture 05 notes, capacity-aware
 * dispatch), or, with batch priority (CS25 Lecture 05 notes, "from language
 * MoE to Vision MoE": high-priority tokens take the slots first), `order`: a
 * permutation of 0..T-1 listing the tokens from the highest priority down,
 * built by the caller.
 * counts[r, e] = claims of rank r on e (pre-capacity); kept[e] =
 * min(sum_r counts[r, e], C); offsets[e] = sum_{e' < e} kept[e'], offsets[N] =
 * total kept rows.  The compact expert-major row of a kept (t, r) is
 * offsets[e] + pos[t, r]. */
void oracle_dispatch_ordered(int64_t T, int32_t N, int32_t k, int32_t C, const int32_t* idx,
                             const int64_t* order, int32_t* pos, uint8_t* drop, int32_t* counts,
                             int32_t* kept, int32_t* offsets) {
    int64_t claims[1024];
    for (int32_t e = 0; e < N; ++e) claims[e] = 0;
    for (int32_t r = 0; r < k; ++r) {
        for (int32_t e = 0; e < N; ++e) counts[r * N + e] = 0;
        for (int64_t q = 0; q < T; ++q) {
            int64_t t = order ? order[q] : q;
            int32_t e = idx[t * k + r];
            int64_t p = claims[e];
            claims[e] = p + 1;
            counts[r * N + e] += 1;
            pos[t * k + r] = (int32_t)p;
            drop[t * k + r] = (uint8_t)(p >= (int64_t)C);
        }
    }
    int64_t acc = 0;
    for (int32_t e = 0; e < N; ++e) {
        int64_t total = claims[e];
        kept[e] = (int32_t)(total < (int64_t)C ? total : (int64_t)C);
        offsets[e] = (int32_t)acc;
        acc += kept[e];
    }
    offsets[N] = (int32_t)acc;
}

/* ---- No-Token-Left-Behind re-routing (top-1) -------------------------------
 * CS25 Lecture 05 notes, "No Token Left Behind": when a token's top-1 expert is
 * full, it is sent on to its second, third ... choice until it gets a slot.
 * Reading: stage 0 is the token-order claim on the first choice; in stage s a
 * token without a slot claims, in token order, on its (s+1)-th expert in the
 * order of its router probabilities probs[t, :] (descending, ties to the lower
 * index), its claim numbered after every claim already made on that expert;
 * it is kept iff that number is below C.  Stages run until every token has a
 * slot or all N choices were tried.  Outputs per token: expert[t] (the expert
 * that kept it; its first choice if none did), gate[t] = probs[t, expert[t]]
 * for a kept token (its first-choice gate if dropped), pos[t] (claim number on
 * expert[t]; C for a dropped token), drop[t]; per expert: counts[e] = every
 * claim made on e over all stages, kept[e] = min(counts[e], C), offsets as in
 * oracle_dispatch.  A kept token's compact row is offsets[e] + pos[t]. */
void oracle_dispatch_ntlb(int64_t T, int32_t N, int32_t C, const float* probs, const float* gate0,
                          int32_t* expert, float* gate, int32_t* pos, uint8_t* drop, int32_t* counts,
                          int32_t* kept, int32_t* offsets) {
    int64_t claims[1024];
    for (int32_t e = 0; e < N; ++e) claims[e] = 0;
    for (int64_t t = 0; t < T; ++t) drop[t] = 1;
    for (int32_t s = 0; s < N; ++s) {
        int64_t left = 0;
        for (int64_t t = 0; t < T; ++t) {
            if (!drop[t]) continue;
            /* the (s+1)-th expert of t: rank experts by probability, ties to the
             * lower index, by counting for each e how many experts precede it */
            const float* p = probs + (size_t)t * N;
            int32_t e_s = -1;
            for (int32_t e = 0; e < N && e_s < 0; ++e) {
                int32_t ahead = 0;
                for (int32_t j = 0; j < N; ++j) {
                    if (p[j] > p[e] || (p[j] == p[e] && j < e)) ++ahead;
                }
                if (ahead == s) e_s = e;
            }
            int64_t c = claims[e_s];
            claims[e_s] = c + 1;
            if (s == 0) expert[t] = e_s;
            if (c < (int64_t)C) {
                drop[t] = 0;
                expert[t] = e_s;
                pos[t] = (int32_t)c;
                gate[t] = p[e_s];
            } else {
                ++left;
            }
        }
        if (left == 0) break;
    }
    for (int64_t t = 0; t < T; ++t) {
        if (drop[t]) {
            pos[t] = C;
            gate[t] = gate0[t];
        }
    }
    int64_t acc = 0;
    for (int32_t e = 0; e < N; ++e) {
        counts[e] = (int32_t)claims[e];
        kept[e] = (int32_t)(claims[e] < (int64_t)C ? claims[e] : (int64_t)C);
        offsets[e] = (int32_t)acc;
        acc += kept[e];
    }
    offsets[N] = (int32_t)acc;
}

void oracle_dispatch(int64_t T, int32_t N, int32_t k, int32_t C, const int32_t* idx,
                     int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept,
                     int32_t* offsets) {
    oracle_dispatch_ordered(T, N, k, C, idx, (const int64_t*)0, pos, drop, counts, kept, offsets);
}

/* ---- One expert on one token -----------------------------------------------
 * ReLU expert:   u = W1 x + b1; a = max(u, 0); y = W2 a + b2.
 * SwiGLU expert: u = W1 x + b1; v = W3 x + b3; a = silu(u) * v; y = W2 a + b2.
 * W1, W3: [d_ff, d]; W2: [d, d_ff] (output-by-input, so W x is a row dot
 * product); biases nullable.  All in double; a is NOT rounded.
 * x: d values (dtype x_dtype); weights and biases: dtype w_dtype.  y: [d]. */
void oracle_expert_ffn(int32_t d, int32_t d_ff, int32_t act,
                       const void* x, int32_t x_dtype, size_t x_off,
                       const void* w1, const void* b1, const void* w3, const void* b3,
                       const void* w2, const void* b2, int32_t w_dtype,
                       size_t w1_off, size_t b1_off, size_t w2_off, size_t b2_off,
                       double* a_scratch, double* y) {
    for (int32_t j = 0; j < d_ff; ++j) {
        double u = 0.0;
        for (int32_t i = 0; i < d; ++i) {
            u += load_elem(w1, w_dtype, w1_off + (size_t)j * d + i) * load_elem(x, x_dtype, x_off + i);
        }
        if (b1) u += load_elem(b1, w_dtype, b1_off + j);
        if (act == ORACLE_RELU) {
            a_scratch[j] = u > 0.0 ? u : 0.0;
        } else {
            double v = 0.0;
            for (int32_t i = 0; i < d; ++i) {
                v += load_elem(w3, w_dtype, w1_off + (size_t)j * d + i) * load_elem(x, x_dtype, x_off + i);
            }
            if (b3) v += load_elem(b3, w_dtype, b1_off + j);
            a_scratch[j] = (u / (1.0 + exp(-u))) * v;
        }
    }
    for (int32_t n = 0; n < d; ++n) {
        double acc = 0.0;
        for (int32_t j = 0; j < d_ff; ++j) {
            acc += load_elem(w2, w_dtype, w2_off + (size_t)n * d_ff + j) * a_scratch[j];
        }
        if (b2) acc += load_elem(b2, w_dtype, b2_off + n);
        y[n] = acc;
    }
}

/* ---- Layer output for a list of tokens --------------------------------------
 * out_t = sum over kept r of g_{t,r} * E_{idx[t,r]}(x_t), in double; zero when
 * no assignment of t is kept (the residual path outside the layer carries a
 * dropped token).  out_exact gets the double value; out_rounded the value
 * rounded once to the output dtype (fp32, or bf16 round-to-nearest-even).
 *
 * x: [T, d]; w1, w3: [N, d_ff, d]; w2: [N, d, d_ff]; b1, b3: [N, d_ff];
 * b2: [N, d].  idx, gate, drop: [T, k] from oracle_router / oracle_dispatch.
 * tokens: the n_tok token indices to evaluate; outputs are [n_tok, d].
 * scratch: d_ff + d doubles. */
void oracle_layer_tokens(int32_t d, int32_t d_ff, int32_t k, int32_t act,
                         const void* x, int32_t x_dtype,
                         const void* w1, const void* b1, const void* w3, const void* b3,
                         const void* w2, const void* b2, int32_t w_dtype,
                         const int32_t* idx, const float* gate, const uint8_t* drop,
                         int64_t n_tok, const int64_t* tokens, int32_t out_dtype,
                         double* scratch, double* out_exact, float* out_rounded) {
    double* a = scratch;
    double* y = scratch + d_ff;
    for (int64_t q = 0; q < n_tok; ++q) {
        int64_t t = tokens[q];
        double* o = out_exact + (size_t)q * d;
        for (int32_t n = 0; n < d; ++n) o[n] = 0.0;
        for (int32_t r = 0; r < k; ++r) {
            if (drop[t * k + r]) continue;
            int32_t e = idx[t * k + r];
            double g = (double)gate[t * k + r];
            oracle_expert_ffn(d, d_ff, act, x, x_dtype, (size_t)t * d,
                              w1, b1, w3, b3, w2, b2, w_dtype,
                              (size_t)e * d_ff * d, (size_t)e * d_ff,
                              (size_t)e * d * d_ff, (size_t)e * d, a, y);
            for (int32_t n = 0; n < d; ++n) o[n] += g * y[n];
        }
        for (int32_t n = 0; n < d; ++n) {
            float v = (float)o[n];
            out_rounded[(size_t)q * d + n] = (out_dtype == ORACLE_BF16) ? oracle_bf16_round(v) : v;
        }
    }
}

/* ---- Un-gated expert outputs in compact expert-major order ------------------
 * ye[row] = E_e(x_t) for each requested compact row, where row = offsets[e] +
 * pos[t, r] for a kept (t, r).  rows_token / rows_expert give (t, e) for each
 * requested row.  Output [n_rows, d] in double. */
void oracle_expert_rows(int32_t d, int32_t d_ff, int32_t act,
                        const void* x, int32_t x_dtype,
                        const void* w1, const void* b1, const void* w3, const void* b3,
                        const void* w2, const void* b2, int32_t w_dtype,
                        int64_t n_rows, const int64_t* rows_token, const int32_t* rows_expert,
                        double* scratch, double* ye) {
    for (int64_t q = 0; q < n_rows; ++q) {
        int64_t t = rows_token[q];
        int32_t e = rows_expert[q];
        oracle_expert_ffn(d, d_ff, act, x, x_dtype, (size_t)t * d,
                          w1, b1, w3, b3, w2, b2, w_dtype,
                          (size_t)e * d_ff * d, (size_t)e * d_ff,
                          (size_t)e * d * d_ff, (size_t)e * d, scratch, ye + (size_t)q * d);
    }
}
