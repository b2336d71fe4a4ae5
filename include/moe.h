/*
 * moe.h -- C ABI of libmoe_b200.so: the forward pass of one sparse
 * Mixture-of-Experts FFN layer (Switch / sparsely-gated MoE) on one B200.
 *
 * The layer, as the pages define it:
 *   router      h = W_r x (+ b_r), fp32;  p = softmax(h)
 *               ("From Switch Transformer to GLaM", section "Dense Scaling vs
 *               MoE"; "Training Stability, Results & Limitations", section 2.1
 *               Selective Precision: the router runs in float32)
 *   top-k gate  k = 1: i* = argmax p, gate p_{i*}  (GLaM page, "Switch
 *               Transformer: making MoE simple");  k = 2: the two largest
 *               logits, gates = softmax over those two logits (CMU 10-423
 *               Lecture 16, section 2.3; GLaM page, "Why GLaM returns to top-2")
 *   capacity    C = floor(k T cf / N) slots per expert (GLaM page, "Expert
 *               Capacity and Token Dropping"; Lecture 16, exercise 3); tokens
 *               claim slots in token order, all first choices before any second
 *               choice (CS25 Lecture 05 notes, capacity-aware dispatch; Lecture
 *               16 section 6.1, GShard rule); an overflowing assignment is
 *               dropped and a token with no kept assignment outputs zero (its
 *               residual connection, outside this layer, carries it)
 *   expert      ReLU: W2 relu(W1 x + b1) + b2 (GLaM page, FFN(x) = W2 s(W1 x));
 *               SwiGLU: W2 (silu(W1 x + b1) * (W3 x + b3)) + b2 (Lecture 16,
 *               section 2.3, Mixtral expert; silu(z) = z / (1 + e^-z))
 *   combine     out_t = sum over kept r of gate_{t,r} * E_{idx[t,r]}(x_t)
 *   aux loss    alpha N sum_i f_i P_i, f_i = fraction of tokens whose top-1
 *               choice is i (before capacity), P_i = mean router probability
 *               (GLaM page, section "Load balancing"; alpha = 1e-2)
 *
 * Beyond the forward: other slot-claim rules (moe_config.priority: batch
 * priority, No-Token-Left-Behind re-routing; moe_dispatch_ntlb), the router
 * z-loss (moe_route_z), one routing group split over several GPUs with one
 * small exchange (moe_expert_counts, moe_claim_base, moe_dispatch_shard,
 * moe_combine_shard, moe_aux_shards), the experts spread over several GPUs
 * with all-to-all dispatch and combine (moe_ep_*), the backward (moe_gate_grad,
 * moe_router_backward, moe_expert_backward), and a dispatch that needs no workspace
 * (moe_dispatch_noalloc).
 *
 * Conventions shared by every entry point
 *   - All array pointers are DEVICE pointers unless stated; the caller owns
 *     every buffer.  The library never allocates or frees memory; the one
 *     exception is the fixed scratch array of moe_dispatch_noalloc (see its
 *     declaration), a static object of the library itself.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Only moe_read_device_status
 *     synchronises.  Calls are stateless apart from the caller's workspace, so
 *     distinct workspaces may be used from distinct threads -- except
 *     moe_dispatch_noalloc, whose calls share one library-wide scratch array
 *     per GPU and must not overlap (see its declaration).
 *   - Layouts (row-major): x, out [T, d_model]; w_r [N, d_model] fp32; b_r [N]
 *     fp32; w1, w3 [N, d_ff, d_model]; w2 [N, d_model, d_ff] ("output x input",
 *     so every product is a row dot product); b1, b3 [N, d_ff]; b2 [N, d_model];
 *     idx, gate, pos, drop [T, k]; counts [k, N]; kept [N]; offsets [N + 1].
 *   - dtype MOE_BF16: x, out, weights and biases are bf16; MOE_F32: all fp32.
 *     The router weights w_r, b_r and the gates are always fp32.
 *   - The compact expert-major row of a kept assignment (t, r) is
 *     offsets[idx[t,r]] + pos[t,r]; rows of expert e are
 *     [offsets[e], offsets[e+1]), in claim order.
 *   - Every pointer must be 16-byte aligned.  Nullable pointers say so.
 *   - Errors come back as a moe_status; invalid arguments are rejected on the
 *     host before anything is launched.  Device-side failures (a bounded wait
 *     that ran out) are latched in the workspace and reported by
 *     moe_read_device_status.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, bad enum */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels handle */
    MOE_ERR_WORKSPACE = 3,     /* workspace pointer null or smaller than required */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    MOE_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (latched) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_RELU = 0, MOE_SWIGLU = 1 } moe_act;

/* Layer shape.  Limits: 0 <= T < 2^28; 1 <= n_experts <= 128; top_k in {1, 2}
 * with top_k <= n_experts; capacity >= 0 (the explicit C; see moe_capacity);
 * d_model, d_ff >= 1; for MOE_BF16, d_model and d_ff multiples of 16.
 * priority selects the order in which assignments claim expert slots:
 *   MOE_ORDER_TOKEN (0): token order (CS25 Lecture 05 notes, capacity-aware
 *     dispatch); every rank-0 claim before any rank-1 claim.
 *   MOE_ORDER_PRIORITY (1): batch priority (CS25 Lecture 05 notes, section on
 *     Vision MoE: with capacity short, the tokens with the highest priority
 *     score take the slots first): tokens by descending first-choice gate
 *     gate[t, 0], ties to the lower token index; still rank-major.  pos is
 *     the claim number in that order.
 *   MOE_ORDER_NTLB (2): No-Token-Left-Behind re-routing, top-1 only (CS25
 *     Lecture 05 notes, "No Token Left Behind": a token whose expert is full
 *     goes on to its next choices until it gets a slot); see
 *     moe_dispatch_ntlb.  moe_forward runs it from the router probabilities
 *     and returns in idx / gate the expert each token finally uses and its
 *     probability.
 * Orders other than MOE_ORDER_TOKEN are not available for the sharded
 * dispatch or moe_dispatch_noalloc, and MOE_ORDER_NTLB not for moe_dispatch
 * (MOE_ERR_UNSUPPORTED). */
typedef enum { MOE_ORDER_TOKEN = 0, MOE_ORDER_PRIORITY = 1, MOE_ORDER_NTLB = 2 } moe_claim_order;
typedef struct {
    int32_t T;
    int32_t d_model;
    int32_t d_ff;
    int32_t n_experts;
    int32_t top_k;
    int32_t capacity;
    int32_t dtype;   /* moe_dtype */
    int32_t act;     /* moe_act */
    float alpha;     /* load-balancing loss weight */
    int32_t priority;  /* moe_claim_order */
} moe_config;

/* Expert capacity C = floor(k * T * cf / N), computed exactly from the binary
 * value of cf (GLaM page, "Expert Capacity and Token Dropping"; CMU 10-423
 * Lecture 16, exercise 3: 1.25 * 2 * 1024 / 8 = 320).  Host-only, no device
 * work.  Returns -1 for T < 0, N < 1, k < 1, cf negative or not finite, or a
 * result above 2^31 - 1. */
int32_t moe_capacity(int64_t T, int32_t n_experts, int32_t top_k, double capacity_factor);

/* Bytes of device workspace every entry point below needs for `cfg` (0 if the
 * config is invalid).  One workspace serves all entry points; it must not be
 * shared by calls that may run concurrently. */
size_t moe_workspace_bytes(const moe_config* cfg);

/* Prepare a workspace for first use: clears the latched device status (the
 * first 256 bytes).  Call once after allocating a workspace, before any other
 * entry point uses it; later calls keep it consistent by themselves.
 * Asynchronous on `stream`. */
int32_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Static description of a status code. */
const char* moe_status_string(int32_t status);

/* Router + load-balancing loss (rows A1, A2, A8 of the hot path).
 * In:  x [T, d] (dtype), w_r [N, d] fp32, b_r [N] fp32 (nullable).
 * Out: idx [T, k] int32 (experts, descending logit, ties to the lower index),
 *      gate [T, k] fp32, probs [T, N] fp32 (nullable: full softmax),
 *      f [N], P [N], aux [1] as fp64 (each nullable).
 * ws: workspace of ws_bytes >= moe_workspace_bytes(cfg). */
int32_t moe_route(const moe_config* cfg, const void* x, const float* w_r, const float* b_r,
                  int32_t* idx, float* gate, float* probs,
                  double* f, double* P, double* aux,
                  void* ws, size_t ws_bytes, void* stream);

/* moe_route plus the router z-loss (CMU 10-423 Lecture 16, section 4.2,
 * "router z-loss", Zoph et al. 2022: a penalty on large router logits; the
 * page's formula is not legible and its experiment reports the router's
 * logsumexp^2, so z is read as the mean over tokens of
 * (log sum_e exp h_{t,e})^2 over the fp32 logits h, unweighted -- the caller
 * applies its coefficient, 0.001 in OLMoE).  Out: z_loss [1] fp64 (nullable);
 * 0 for T = 0.  Per-token values are summed in fp64 in a fixed order.  The
 * other arguments and outputs are those of moe_route. */
int32_t moe_route_z(const moe_config* cfg, const void* x, const float* w_r, const float* b_r,
                    int32_t* idx, float* gate, float* probs,
                    double* f, double* P, double* aux, double* z_loss,
                    void* ws, size_t ws_bytes, void* stream);

/* Gradient of L with respect to the gates, from the upstream dL/dout and the
 * un-gated expert outputs (out_t = sum_r gate_{t,r} E_{idx[t,r]}(x_t)):
 * dgate[t, r] = <dout_t, ye[offsets[idx[t,r]] + pos[t,r]]> for a kept
 * assignment, 0 for a dropped one; fp32 accumulation.  In: dout [T, d]
 * (dtype), ye [R, d] (dtype; moe_expert_ffn's output), idx, pos, drop [T, k],
 * offsets [N + 1].  Out: dgate [T, k] fp32 -- the input of
 * moe_router_backward. */
int32_t moe_gate_grad(const moe_config* cfg, const void* dout, const void* ye, const int32_t* idx,
                      const int32_t* pos, const uint8_t* drop, const int32_t* offsets, float* dgate,
                      void* stream);

/* Router backward (fp32): gradients of L = sum_{t,r} dgate[t,r] gate[t,r] +
 * L_aux with respect to the router logits, W_r, b_r and the router input x.
 * Gate path ("From Switch Transformer to GLaM": top-1 gate p_{i*}, top-2 the
 * softmax over the two kept logits; the expert choice has no gradient) and
 * the load-balancing loss with f held constant (CMU 10-423 Lecture 16,
 * section 4.2: dL_aux/dp_{t,i} = alpha N f_i / T, alpha = cfg->alpha).
 * In:  x [T, d] (dtype), w_r [N, d], probs [T, N] (moe_route's full softmax),
 *      idx, gate [T, k] (moe_route's), f [N] fp64 (moe_route's), dgate [T, k]
 *      fp32 (dL/dgate: <dL/dout_t, E_{idx}(x_t)> for a kept assignment, 0
 *      for a dropped one).
 * Out: dh [T, N] fp32 (dL/dh); dw_r [N, d], db_r [N], dx [T, d] fp32 (each
 *      nullable; dx is the router's part of dL/dx).  Sums over tokens run per
 *      512-token chunk in fp32 and over chunks in fp64, in a fixed order. */
int32_t moe_router_backward(const moe_config* cfg, const void* x, const float* w_r, const float* probs,
                            const int32_t* idx, const float* gate, const double* f, const float* dgate,
                            float* dh, float* dw_r, float* db_r, float* dx,
                            void* ws, size_t ws_bytes, void* stream);

/* Backward of the expert FFN (bf16, on the tensor cores): gradients of
 * L = sum_t <dout_t, out_t> through the combine, the expert FFNs and their
 * weights ("From Switch Transformer to GLaM", FFN(x) = W2 s(W1 x); CMU 10-423
 * Lecture 16, section 2.3, SwiGLU expert), with the gates held fixed (their
 * gradient is moe_gate_grad's).  For a kept row r of expert e (token t, gate
 * g): dY = g dout_t; dA = dY W2[e]; dU = dA * relu'(u) (SwiGLU: dG = dA * up *
 * silu'(gate pre-activation), dUp = dA * silu(gate pre-activation));
 * dx_t += dU W1[e] (+ dUp W3[e]); dW1[e] = sum_r dU^T x, dW3[e] = sum_r dUp^T x,
 * dW2[e] = sum_r dY^T a; db1, db3, db2 the column sums of dU, dUp, dY.  The
 * first GEMM is recomputed from xe (its activations are not kept by the
 * forward).  bf16 operands, fp32 accumulation; gradients are fp32.
 * In:  xe [R, d], offsets [N + 1], row_token, row_gate [R] (moe_dispatch's),
 *      idx, pos, drop [T, k], dout [T, d] bf16, w1, w3 [N, d_ff, d], w2
 *      [N, d, d_ff], b1, b3 [N, d_ff] (nullable).
 * Out: dx [T, d] fp32 (the expert part of dL/dx; 0 for a token with no kept
 *      assignment), dw1, dw3 [N, d_ff, d], dw2 [N, d, d_ff], db1, db3 [N, d_ff],
 *      db2 [N, d] fp32 (each nullable; experts without rows get zeros).
 * ws: moe_expert_backward_workspace_bytes(cfg) bytes, moe_workspace_init'ed.
 * MOE_ERR_UNSUPPORTED for MOE_F32, and for SwiGLU with d_ff not a multiple of 64. */
size_t moe_expert_backward_workspace_bytes(const moe_config* cfg);
int32_t moe_expert_backward(const moe_config* cfg, const void* xe, const int32_t* offsets, const int32_t* row_token,
                            const float* row_gate, const int32_t* idx, const int32_t* pos, const uint8_t* drop,
                            const void* dout, const void* w1, const void* b1, const void* w3, const void* b3,
                            const void* w2, float* dx, float* dw1, float* db1, float* dw3, float* db3, float* dw2,
                            float* db2, void* ws, size_t ws_bytes, void* stream);

/* Capacity-limited dispatch (row A3 and the gather of A4).
 * In:  x [T, d] (dtype; nullable when xe is NULL), idx [T, k], gate [T, k].
 * Out: pos [T, k] int32 (claim number of the assignment on its expert: all
 *      rank-0 claims in token order, then the rank-1 claims), drop [T, k] uint8
 *      (1 iff pos >= C), counts [k, N] (claims per rank before capacity),
 *      kept [N] = min(sum_r counts[r][e], C), offsets [N + 1] (exclusive prefix
 *      of kept), row_token [R] / row_gate [R] (token and gate of every compact
 *      row, R = offsets[N]), xe [R, d] (dtype; the gathered rows; nullable).
 *      The row_* and xe buffers must hold min(k T, N C) rows. */
int32_t moe_dispatch(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate,
                     int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept,
                     int32_t* offsets, int32_t* row_token, float* row_gate, void* xe,
                     void* ws, size_t ws_bytes, void* stream);

/* No-Token-Left-Behind dispatch (top-1; cfg->priority must be MOE_ORDER_NTLB).
 * Stage 0 is the token-order claim on each token's first expert; in stage s
 * every token still without a slot claims, in token order, on its (s+1)-th
 * expert by router probability (descending, ties to the lower index), its
 * claim numbered after all earlier claims on that expert; it is kept iff the
 * number is below C.  Stages run until all N choices were tried.
 * In:  probs [T, N] fp32 (moe_route's full softmax), x [T, d] (nullable when
 *      xe is NULL).
 * Out: expert [T] int32 (the expert that kept the token; its first choice if
 *      none did), gate [T] fp32 (probs[t, expert[t]]), pos [T] (claim number
 *      on expert[t]; C if dropped), drop [T], counts [N] (claims on each
 *      expert over all stages), kept [N] = min(counts, C), offsets [N + 1],
 *      row_token / row_gate / xe as moe_dispatch (row offsets[e] + pos).
 * Cost: one cooperative kernel runs the stages (one grid barrier each) and
 * stops after the first stage that leaves no token unplaced, then the gather. */
int32_t moe_dispatch_ntlb(const moe_config* cfg, const void* x, const float* probs,
                          int32_t* expert, float* gate, int32_t* pos, uint8_t* drop,
                          int32_t* counts, int32_t* kept, int32_t* offsets,
                          int32_t* row_token, float* row_gate, void* xe,
                          void* ws, size_t ws_bytes, void* stream);

/* ---- One routing group split over several shards (one per GPU) ------------
 * Capacity is defined per routing group, and claims follow token order over the
 * whole group (CS25 Lecture 05 notes, capacity-aware dispatch).  When a group's
 * tokens are split into contiguous shards, shard s computes exactly what a
 * single call over the whole group computes for its tokens if it knows, per
 * (rank, expert), how many claims come before its own:
 *   1. moe_route on the shard;  2. moe_expert_counts -> this shard's claims
 *   counts_s[k][N];  3. every shard gathers all shards' counts into
 *   [S][k][N] (one small all-gather, the only exchange);  4. moe_claim_base;
 *   5. moe_dispatch_shard;  then moe_expert_ffn on the shard's own compact
 *   rows and moe_combine_shard;  6. the aux loss over the group with moe_aux_shards from
 *   every shard's f, P and token count (one more small all-gather).
 * Routing integers and outputs are then identical to the single call. */

/* Claims of this shard: counts[r][e] = number of tokens whose rank-r choice is
 * e (before capacity).  In: idx [T, k].  Out: counts [k, N] int32. */
int32_t moe_expert_counts(const moe_config* cfg, const int32_t* idx, int32_t* counts, void* stream);

/* Claim base of shard `shard` among n_shards contiguous shards (shard order =
 * token order).  In: shard_counts [n_shards][top_k][n_experts] int32 (device).
 * Out: claim_base [top_k][n_experts] int32 (device):
 *   claim_base[0][e] = rank-0 claims on e by earlier shards,
 *   claim_base[1][e] = every shard's rank-0 claims on e + rank-1 claims on e
 *                      by earlier shards. */
int32_t moe_claim_base(const int32_t* shard_counts, int32_t n_shards, int32_t shard, int32_t top_k,
                       int32_t n_experts, int32_t* claim_base, void* stream);

/* moe_dispatch for one shard of a routing group: cfg->T is the shard's token
 * count, cfg->capacity the group's C.  pos are the group-wide claim numbers
 * (claim_base + the shard's own claim order), drop = pos >= C; counts are the
 * shard's own claims; kept/offsets/row_token/row_gate/xe describe the shard's
 * kept assignments, in the order moe_dispatch would give them. */
int32_t moe_dispatch_shard(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate,
                           const int32_t* claim_base, int32_t* pos, uint8_t* drop, int32_t* counts,
                           int32_t* kept, int32_t* offsets, int32_t* row_token, float* row_gate, void* xe,
                           void* ws, size_t ws_bytes, void* stream);

/* Load-balancing loss of a routing group from its shards (GLaM page, Load
 * balancing): f = sum_s T_s f_s / sum_s T_s, likewise P, aux = alpha N sum f P,
 * in fp64 in shard order.  In: shard_tokens [S] int64, f_all, P_all [S][N]
 * fp64 (each shard's moe_route outputs), all device.  Out: f, P [N], aux [1]
 * fp64 (each nullable). */
int32_t moe_aux_shards(int32_t n_shards, int32_t n_experts, const int64_t* shard_tokens, const double* f_all,
                       const double* P_all, float alpha, double* f, double* P, double* aux, void* stream);

/* Grouped expert FFN over the compact rows (rows A5, A6).
 * In:  xe [R, d] (dtype) with R = offsets[N]; offsets [N + 1]; w1, w2 and
 *      (SwiGLU) w3; b1, b3, b2 nullable.
 * Out: ye [R, d] (dtype): the un-gated expert output of every row. */
int32_t moe_expert_ffn(const moe_config* cfg, const void* xe, const int32_t* offsets,
                       const void* w1, const void* b1, const void* w3, const void* b3,
                       const void* w2, const void* b2, void* ye,
                       void* ws, size_t ws_bytes, void* stream);

/* Gate-scaled combine back to token order (row A7).
 * out[t] = sum over r with drop[t,r] == 0 of gate[t,r] * ye[offsets[idx[t,r]] +
 * pos[t,r]], accumulated in fp32 and rounded once; zero if every assignment of
 * t was dropped.  In: ye [R, d], idx, pos, drop, gate [T, k], offsets [N + 1].
 * Out: out [T, d] (dtype). */
int32_t moe_combine(const moe_config* cfg, const void* ye, const int32_t* idx,
                    const int32_t* pos, const uint8_t* drop, const float* gate,
                    const int32_t* offsets, void* out, void* stream);

/* moe_combine for one shard of a routing group, after moe_dispatch_shard:
 * pos are group-wide claim numbers, and the row of a kept claim p on expert e
 * is offsets[e] + p - claim_base[0][e] for rank 0 and offsets[e] +
 * kept0[e] + p - claim_base[1][e] for rank 1, kept0[e] = how many of the
 * shard's rank-0 claims on e fall below C.  In: claim_base [k, N] (from
 * moe_claim_base) and counts [k, N] (the shard's own, from
 * moe_dispatch_shard), both required; the rest as moe_combine. */
int32_t moe_combine_shard(const moe_config* cfg, const void* ye, const int32_t* idx,
                          const int32_t* pos, const uint8_t* drop, const float* gate,
                          const int32_t* offsets, const int32_t* claim_base,
                          const int32_t* counts, void* out, void* stream);

/* The whole layer forward in one call (rows A1-A8), fused where it pays:
 * the top-1 bf16 path scatters gate * E(x) straight from the second GEMM's
 * epilogue into out.
 * In:  x, w_r, b_r (nullable), w1, b1 (nullable), w3 (SwiGLU), b3 (nullable),
 *      w2, b2 (nullable).
 * Out: out [T, d] (required); idx, gate, pos, drop, counts, kept, offsets, f, P,
 *      aux: each nullable (when NULL the value stays in the workspace). */
int32_t moe_forward(const moe_config* cfg, const void* x, const float* w_r, const float* b_r,
                    const void* w1, const void* b1, const void* w3, const void* b3,
                    const void* w2, const void* b2, void* out,
                    int32_t* idx, float* gate, int32_t* pos, uint8_t* drop,
                    int32_t* counts, int32_t* kept, int32_t* offsets,
                    double* f, double* P, double* aux,
                    void* ws, size_t ws_bytes, void* stream);

/* moe_forward, plus stage timing for profiling: `events` points to 6 cudaEvent_t
 * handles (passed as void*, created by the caller; any entry may be NULL) that
 * are recorded on `stream` at the stage boundaries: [0] before the router,
 * [1] after the router and aux loss, [2] after the dispatch and gather, [3]
 * after the first expert GEMM, [4] after the second expert GEMM, [5] after the
 * combine (equal to [4] on the fused top-1 path).  events == NULL behaves as
 * moe_forward.  The kernels launched are identical to moe_forward's. */
int32_t moe_forward_events(const moe_config* cfg, const void* x, const float* w_r, const float* b_r,
                           const void* w1, const void* b1, const void* w3, const void* b3,
                           const void* w2, const void* b2, void* out,
                           int32_t* idx, float* gate, int32_t* pos, uint8_t* drop,
                           int32_t* counts, int32_t* kept, int32_t* offsets,
                           double* f, double* P, double* aux,
                           void* ws, size_t ws_bytes, void* stream, void* const* events);

/* ---- Expert parallelism: the experts spread over several GPUs -------------
 * "From Switch Transformer to GLaM", section All-to-All: the experts of a layer
 * live on different devices; a dispatch all-to-all moves every token from the
 * device that holds it to the device of its expert, the experts run there, and
 * a combine all-to-all brings the outputs back.  CMU 10-423 Lecture 16,
 * section 6.2 and exercise 4: this moves 2 * T_g * k * d * 2 B * (G - 1) / G
 * per GPU per layer (bf16), about 235 MB for Mixtral-size layers on 8 GPUs.
 *
 * G GPUs (n_ranks), N experts, E = N / G per GPU: expert e lives on GPU e / E
 * and each GPU holds only the weights of its own E experts.  Every GPU keeps
 * its own batch of T tokens as its own routing group (its capacity C, its
 * aux loss), so its output equals the one-GPU layer forward of its batch.
 * One forward, per GPU g:
 *   1. moe_route, then moe_dispatch with xe = NULL (slot claim and row maps;
 *      the gather is fused into step 4);
 *   2. all-gather every GPU's kept [N] into kept_all [G][N] (NCCL, 512 B);
 *   3. moe_ep_layout;
 *   4. moe_ep_dispatch: x rows into their experts' GPUs (peer stores);
 *   5. barrier across the GPUs (e.g. a one-element NCCL all-reduce on the
 *      stream): every GPU's rows have landed;
 *   6. moe_ep_expert_ffn on the received rows: the second GEMM's epilogue
 *      stores every result row straight into its source GPU's buffer;
 *   7. barrier again; 8. top-2 only: moe_combine on the GPU's own ye.
 * Peer buffers are reached through device pointers the caller maps (CUDA IPC);
 * "pointer tables" below are DEVICE arrays of G device pointers, entry s
 * addressing GPU s's buffer (this GPU's own entry its own buffer).  Only plain
 * loads from local memory and plain stores to peer memory cross GPUs. */

/* Receive rows each GPU must provide (recv_x [R, d], recv_rank / recv_row /
 * recv_gate [R]): R = G * min(k T, E C) (k counted at most E); -1 if invalid
 * (N not a multiple of n_ranks, or the config is invalid). */
int64_t moe_ep_recv_rows(const moe_config* cfg, int32_t n_ranks);

/* Workspace bytes of moe_ep_expert_ffn (0 if invalid). */
size_t moe_ep_workspace_bytes(const moe_config* cfg, int32_t n_ranks);

/* Where rows land.  In: kept_all [G][N] int32 (every GPU's moe_dispatch kept,
 * GPU order).  Out: dst_start [N] (GPU `rank` as a source: its rows of expert
 * e go to rows dst_start[e] ... of GPU e / E's receive buffer) and
 * recv_offsets [E + 1] (GPU `rank` as a receiver: rows of its local expert j
 * are [recv_offsets[j], recv_offsets[j + 1]), source GPU 0's rows first, each
 * source's in its own claim order). */
int32_t moe_ep_layout(int32_t n_ranks, int32_t rank, int32_t n_experts, const int32_t* kept_all,
                      int32_t* dst_start, int32_t* recv_offsets, void* stream);

/* Dispatch all-to-all with the gather fused in: for every kept row r of this
 * GPU (moe_dispatch's offsets / row_token / row_gate), x[row_token[r]] is
 * stored into row dst_start[e] + r - offsets[e] of recv_x[e / E], with its
 * return address: recv_rank = rank, recv_row = the token (top-1) or r (top-2),
 * recv_gate = row_gate[r].  Top-1: also zeroes out [T, d] rows of dropped
 * tokens (drop [T, 1]); out is ignored for top-2.  cfg is this GPU's layer
 * (its T, the total N, k, C, dtype).  recv_x, recv_rank, recv_row, recv_gate:
 * pointer tables [G]. */
int32_t moe_ep_dispatch(const moe_config* cfg, int32_t n_ranks, int32_t rank, const void* x,
                        const int32_t* offsets, const int32_t* row_token, const float* row_gate,
                        const uint8_t* drop, const int32_t* dst_start, void* const* recv_x,
                        int32_t* const* recv_rank, int32_t* const* recv_row, float* const* recv_gate,
                        void* out, void* stream);

/* The local experts on the received rows, results sent back.  In: recv_x,
 * recv_offsets [E + 1], recv_rank, recv_row, recv_gate (this GPU's receive
 * buffers, filled by every GPU's moe_ep_dispatch); w1, w3 [E, d_ff, d], w2
 * [E, d, d_ff], b1, b3 [E, d_ff], b2 [E, d] (nullable): this GPU's experts only.
 * out_ptrs: pointer table [G]; top-1: every GPU's out [T, d], row recv_row
 * receives recv_gate * E(x); top-2: every GPU's ye [min(k T, N C), d], row
 * recv_row receives E(x) (then moe_combine on that GPU).  bf16: stored from the
 * second GEMM's epilogue; fp32: after the expert FFN, by a copy kernel.
 * ws: moe_ep_workspace_bytes(cfg, n_ranks) bytes, moe_workspace_init'ed. */
int32_t moe_ep_expert_ffn(const moe_config* cfg, int32_t n_ranks, const void* recv_x, const int32_t* recv_offsets,
                          const void* w1, const void* b1, const void* w3, const void* b3, const void* w2,
                          const void* b2, const int32_t* recv_rank, const int32_t* recv_row,
                          const float* recv_gate, void* const* out_ptrs, void* ws, size_t ws_bytes,
                          void* stream);

/* Synchronise `stream`, then return the device status latched in the
 * workspace: MOE_OK, or MOE_ERR_TIMEOUT if a bounded device-side wait gave up
 * during an earlier call on this workspace.  The outputs of such a call are
 * undefined; the CUDA context stays usable.  A non-OK status is cleared by the
 * read, together with the workspace's per-call counters, so the workspace is
 * ready for the next call. */
int32_t moe_read_device_status(void* ws, void* stream);

/* moe_dispatch without a workspace, for callers that cannot allocate device
 * memory when they call the layer: plugin interfaces that give a kernel only
 * its input and output tensors, and serving runtimes that reserve all device
 * memory at start-up and allow no cudaMalloc later (it synchronises the device
 * and can fail once memory is fragmented).  The pages have no counterpart to
 * this entry point; it computes exactly what moe_dispatch computes, with the
 * same launches.
 * Scratch: the dispatch scan's flags and counters live in a fixed-size
 * __device__ array inside the library (about 256 KB, held on every GPU that
 * loads the library until the process exits).  Limit: T <= 262144 tokens;
 * larger T returns MOE_ERR_UNSUPPORTED before anything is launched.  The call
 * allocates nothing and frees nothing.
 * The array is shared by every call and keeps the last call's contents (each
 * call clears what it uses first), so calls whose work can overlap on one GPU
 * -- different streams, or different host threads on the same device -- race
 * and must be serialised by the caller.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture starts.  The address is kept
 * for the life of the process: do not reset the device (cudaDeviceReset)
 * between calls.
 * Arguments are those of moe_dispatch, without ws/ws_bytes, plus
 * status: device int32 (nullable) that receives this call's device-side status
 * (MOE_OK, or MOE_ERR_TIMEOUT if the scan's bounded wait gave up). */
int32_t moe_dispatch_noalloc(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate,
                             int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept,
                             int32_t* offsets, int32_t* row_token, float* row_gate, void* xe,
                             int32_t* status, void* stream);

/* Test hook (not part of the layer): launch one block of the dispatch scan's
 * look-back in isolation, waiting on a predecessor that never publishes, with a
 * wait limit of `limit_ns` nanoseconds.  The wait gives up, latches
 * MOE_ERR_TIMEOUT in the workspace and returns; read it back with
 * moe_read_device_status. */
int32_t moe_test_lookback_timeout(void* ws, size_t ws_bytes, int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
