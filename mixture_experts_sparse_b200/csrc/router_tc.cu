// Router of the MoE layer on the tensor cores, for bf16 activations.
//
// Same definition as the FP32-pipe router (router.cu): fp32 logits h = W_r x
// (+ b_r), softmax, top-k with ties to the lower index, gates, and per-tile
// load-balancing partials ("From Switch Transformer to GLaM", "Dense Scaling vs
// MoE", "Switch Transformer: making MoE simple", "Load balancing"; CMU 10-423
// Lecture 16, section 2.3; "Training Stability, Results & Limitations", 2.1:
// the router is an fp32 computation on the up-cast bf16 input).
//
// Why the tensor cores can do an fp32 router here: x is bf16, so every x value
// is exact in bf16, and each fp32 router weight w splits exactly into three
// bf16 parts w = w0 + w1 + w2 (8 + 8 + 8 significand bits; w0 = bf16(w),
// w1 = bf16(w - w0), w2 = w - w0 - w1).  Every product x * w_p is exact in fp32,
// and the tensor core accumulates them in fp32, so
//   h = sum_j x_j w0_j + sum_j x_j w1_j + sum_j x_j w2_j
// is the fp32 dot product up to accumulation rounding -- 3 NP columns of bf16
// MMA per K step.  With 3 NP <= 256 the three parts are adjacent rows of one B
// tile, so a single MMA of N = 3 NP produces the three partial logits side by
// side in TMEM (the epilogue adds them in fp32); with NP = 128, an MMA of
// N = 256 (parts 0 and 1) and one of N = 128 (part 2, added to part 1's
// block) -- an MMA costs about the same issue time at N = 128 as at N = 256,
// so two instructions per K step instead of three.  The tensor core's fp32
// accumulation truncates, so its error grows with the number of MMAs summed
// into one accumulator at the logits' scale; the K loop is therefore cut into
// G groups of at most 64 such MMAs, each group in its own TMEM column block,
// and the epilogue adds the partial logits in fp32 with round-to-nearest in a
// fixed order.  The router then costs about one read of x from HBM instead of
// 2 d N FP32-pipe FLOPs per token.
//
// Kernel: persistent CTA pairs (clusters of two), 192 threads per CTA.  A
// pair owns a 256-token tile and issues cta_group::2 MMAs (M = 256 tokens, 128
// per CTA): each CTA loads its own 128 x 64 x tile and half of the three W
// parts' rows, so the W bytes streamed per token are half those of a one-CTA
// tile and more stages fit.  Warp 0 TMA producer (128-byte swizzle; both
// CTAs' loads complete on the leader's barrier), warp 1 TMEM allocator + MMA
// issuer (the leader's), warps 2-5 epilogue with one thread per token of its
// own CTA: the thread holds its token's NP logits (tcgen05.ld), computes max,
// softmax, top-1/top-2 and the gate in registers, and writes idx/gate (and
// probs).  Per-tile sums of p are reduced across each warp's lanes with a
// fixed shuffle tree that leaves every lane the sums of NP/32 experts (kept in
// registers over the CTA's tiles), then over the four warps in a fixed order,
// so the aux loss is deterministic and no shared memory holds per-token sums.
#include "tc_common.cuh"

namespace moe {
using namespace tc;
namespace {

constexpr int RT_THREADS = 192;
constexpr int RT_BM = 128;       // tokens per CTA (256 per pair)
constexpr int RT_BK = 64;

template <int NP>
struct RtShape {
    // merged: one MMA of N = 3 NP covers the three W parts and leaves three
    // partial-logit blocks side by side in TMEM; the pair's leader holds W rows
    // [0, 3 NP / 2) of the stacked parts, the peer rows [3 NP / 2, 3 NP).
    // Otherwise (NP = 128) two MMAs per K slice: one of N = 256 over parts 0
    // and 1 (the leader holds part 0, the peer part 1) into column blocks 0 and
    // 1, and one of N = 128 over part 2 (NP / 2 rows per CTA) that accumulates
    // into block 1 -- parts 1 and 2 are 2^-8 and 2^-16 of w, so their shared
    // accumulator stays 2^8 below the logits and its truncation error with it.
    static constexpr bool MERGED = 3 * NP <= 256;
    // K boxes (64 deep) per pipeline stage: two when merged (8 MMAs per
    // barrier round trip), one otherwise (two MMAs per K slice, 8 per stage)
    static constexpr int KSUB = MERGED ? 2 : 1;
    static constexpr int A_SUB = RT_BM * RT_BK * 2;             // one x box
    static constexpr int A_BYTES = A_SUB * KSUB;
    static constexpr int P_BYTES = (NP / 2) * RT_BK * 2;       // this CTA's half of one W part, one box
    static constexpr int W_BOX = MERGED ? 3 * NP / 2 : NP / 2;   // rows per W load
    static constexpr int W_SUB = MERGED ? W_BOX * RT_BK * 2 : 3 * P_BYTES;   // W bytes per K box
    static constexpr int STAGE_BYTES = A_BYTES + KSUB * W_SUB;
    // as many stages as fit (the router is bound by the x bytes in flight)
    static constexpr int STAGES = (200 * 1024) / STAGE_BYTES < 12 ? (200 * 1024) / STAGE_BYTES : 12;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
    static constexpr int BLOCKS = MERGED ? 3 : 2;              // partial-logit column blocks per accumulator
    static constexpr int ACC_COLS = BLOCKS * NP;               // TMEM columns per K-group accumulator
    static constexpr int TMEM_COLS = 512;                      // buffers x G groups x ACC_COLS
    // per stage, MMAs into the full-scale block (part 0's sums)
    static constexpr int MMA_PER_KB = KSUB * (RT_BK / 16);
    static constexpr int KB_PER_GROUP = 64 / MMA_PER_KB;       // <= 64 MMAs per full-scale accumulator
    static_assert(STAGE_BYTES % 1024 == 0, "1024-byte aligned stages");
    static_assert(STAGES >= 2, "double-buffered stages");
    static constexpr int PER_LANE = NP / 32;   // experts whose warp sums of p a lane keeps
};

// Warp transpose-reduce: every lane holds NP values; after log2(32) halving
// steps (partner = lane ^ 16, 8, 4, 2, 1; the lower-bit lane keeps the lower
// half and adds the partner's copy of it) lane l holds the sums over the 32
// lanes of experts [l NP / 32, (l + 1) NP / 32), in a fixed order.
template <int NP>
__device__ __forceinline__ void warp_transpose_sum(float (&v)[NP], int lane, float (&out)[NP / 32]) {
    float a[NP / 2];
#pragma unroll
    for (int j = 0; j < NP / 2; ++j) {
        const bool hi = lane & 16;
        const float send = hi ? v[j] : v[j + NP / 2];
        const float keep = hi ? v[j + NP / 2] : v[j];
        a[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int o = 8, w = NP / 4; o >= 1; o >>= 1, w >>= 1) {
#pragma unroll
        for (int j = 0; j < w; ++j) {
            const bool hi = lane & o;
            const float send = hi ? a[j] : a[j + w];
            const float keep = hi ? a[j + w] : a[j];
            a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int j = 0; j < NP / 32; ++j) out[j] = a[j];
}

struct RtParams {
    int64_t T;
    int N, k, d;
    int groups;   // K groups with separate accumulators
    int nbuf;     // accumulator buffers (2: the epilogue overlaps the next tile's MMAs)
    int kb_per_group;
    const float* b_r;
    int32_t* idx;
    float* gate;
    float* probs;
    int32_t* part_cnt;    // [N, Gp] per-CTA top-1 counts (Gp = gridDim.x rounded up to 4)
    float* part_psum;     // [N, Gp] per-CTA sums of p
    double* f;            // outputs of the aux loss (nullable)
    double* P;
    double* aux;
    float alpha;
    int32_t* ticket;      // finished-CTA counter, 0 between calls
    int32_t* status;
    int defer_aux;        // 1: the partials are reduced later (aux_reduce_block elsewhere)
    double* part_z;       // [Gp] per-CTA sums of lse^2 (null: no z-loss)
    double* z;
    long long limit_ns;
};

// Fixed-order tree reductions over a thread's NP values (short dependency
// chains; a serial chain over NP values is latency-bound with one warp per SM
// sub-partition).
// (excl: an index whose value is treated as -inf; -1 for none)
template <int NP>
__device__ __forceinline__ float tree_max(const float (&v)[NP], int excl = -1) {
    float t[NP / 2];
#pragma unroll
    for (int j = 0; j < NP / 2; ++j)
        t[j] = fmaxf(2 * j == excl ? -INFINITY : v[2 * j], 2 * j + 1 == excl ? -INFINITY : v[2 * j + 1]);
#pragma unroll
    for (int w = NP / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
    return t[0];
}
template <int NP>
__device__ __forceinline__ float tree_sum(const float (&v)[NP]) {
    float t[NP / 2];
#pragma unroll
    for (int j = 0; j < NP / 2; ++j) t[j] = v[2 * j] + v[2 * j + 1];
#pragma unroll
    for (int w = NP / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) t[j] = t[j] + t[j + w];
    return t[0];
}
// lowest index e with v[e] == m (NP if none)
template <int NP>
__device__ __forceinline__ int tree_first(const float (&v)[NP], float m, int excl = -1) {
    int t[NP / 2];
#pragma unroll
    for (int j = 0; j < NP / 2; ++j)
        t[j] = (v[2 * j] == m && 2 * j != excl) ? 2 * j : ((v[2 * j + 1] == m && 2 * j + 1 != excl) ? 2 * j + 1 : NP);
#pragma unroll
    for (int w = NP / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) t[j] = min(t[j], t[j + w]);
    return t[0];
}

template <int NP>
__global__ void __launch_bounds__(RT_THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, const RtParams p) {
    using S = RtShape<NP>;
    // merged: N = 3 NP; otherwise N = 256 (parts 0, 1) and N = 128 (part 2)
    constexpr uint32_t IDESC = idesc_bf16_f32(2 * RT_BM, S::MERGED ? S::ACC_COLS : 2 * NP);
    constexpr uint32_t IDESC2 = idesc_bf16_f32(2 * RT_BM, NP);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ float s_wsum[4][NP];    // per epilogue warp: sums of p over its tokens
    __shared__ __align__(8) uint64_t full_bar[S::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[S::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_hist[NP];
    __shared__ __align__(16) float s_bias[NP];   // b_r, 0 without a bias, -inf for padding experts
    __shared__ double s_z[128];    // per epilogue thread: sum of lse^2 over its tokens
    __shared__ int s_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();   // 0 = the pair's leader
    const bool leader = rank == 0;
    const int first_tile = (int)cluster_id_x();
    const int tile_step = (int)ncluster_x();
    if (tid == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull_bar[a]), 1);
            mbar_init(smem_u32(&tempty_bar[a]), 256);   // both CTAs' epilogue threads
        }
        mbar_init(smem_u32(&done_bar), 1);
        s_abort = 0;
        mbar_fence_init();
    }
    for (int e = tid; e < NP; e += RT_THREADS) s_hist[e] = 0;
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
    }
    if (warp == 1) tmem_alloc_pair(&s_tmem, S::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // the peer's barriers exist before any cross-CTA signal
    tc_fence_after();
    pdl_wait();       // x, the W split and the workspace are ready from here on
    pdl_launch();
    for (int e = tid; e < NP; e += RT_THREADS)
        s_bias[e] = e < p.N ? (p.b_r ? p.b_r[e] : 0.f) : -INFINITY;   // padding experts never win
    __syncthreads();

    const uint32_t tmem_base = s_tmem;
    const int ntiles = (int)((p.T + 2 * RT_BM - 1) / (2 * RT_BM));
    const int nkb = (p.d + S::KSUB * RT_BK - 1) / (S::KSUB * RT_BK);   // stages per tile
    const Waiter w{&s_abort, p.status, p.limit_ns};

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int last_par[S::STAGES];
#pragma unroll
            for (int s = 0; s < S::STAGES; ++s) last_par[s] = -1;
            bool ok = true;
            for (int tile = first_tile; tile < ntiles && ok; tile += tile_step) {
                const int xrow = tile * 2 * RT_BM + (int)rank * RT_BM;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(smem_u32(&empty_bar[stage]), phase ^ 1u, w)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t fb_leader = map_to_rank(fb, 0);
                    const uint32_t a_dst = smem_u32(smem + stage * S::STAGE_BYTES);
                    if (leader) mbar_expect_tx(fb, 2 * S::STAGE_BYTES);   // both CTAs' bytes
#pragma unroll
                    for (int j = 0; j < S::KSUB; ++j) {
                        const int k0 = (kb * S::KSUB + j) * RT_BK;
                        const uint32_t w_dst = a_dst + S::A_BYTES + j * S::W_SUB;
                        tma_load_2d_pair(a_dst + j * S::A_SUB, &tmX, fb_leader, k0, xrow);
                        if constexpr (S::MERGED) {
                            tma_load_2d_pair(w_dst, &tmW, fb_leader, k0, (int)rank * S::W_BOX);
                        } else {   // this CTA's part (leader 0, peer 1), all NP rows; then its half of part 2
                            tma_load_2d_pair(w_dst, &tmW, fb_leader, k0, (int)rank * NP);
                            tma_load_2d_pair(w_dst + S::P_BYTES, &tmW, fb_leader, k0, (int)rank * NP + S::W_BOX);
                            tma_load_2d_pair(w_dst + 2 * S::P_BYTES, &tmW, fb_leader, k0, 2 * NP + (int)rank * S::W_BOX);
                        }
                    }
                    last_par[stage] = (int)phase;
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the leader's MMA released every stage this thread filled, which it
            // does only after the stage's bytes (both CTAs') arrived
            for (int s = 0; s < S::STAGES; ++s)
                if (last_par[s] >= 0) drain_bar(smem_u32(&empty_bar[s]), (uint32_t)last_par[s], p.limit_ns, p.status);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true, issued = false;
            const uint64_t desc0 = umma_desc(smem_u32(smem));
            for (int tile = first_tile; tile < ntiles && ok; tile += tile_step, ++it) {
                const int acc = p.nbuf == 2 ? (it & 1) : 0;
                const uint32_t acc_par = (uint32_t)(p.nbuf == 2 ? ((it >> 1) & 1) : (it & 1));
                if (!wait_bar(smem_u32(&tempty_bar[acc]), acc_par ^ 1u, w)) break;
                tc_fence_after();
                int g = 0, kin = 0;   // K group and k-block inside it (no division on the issue path)
                for (int kb = 0; kb < nkb; ++kb) {
                    const bool first = kin == 0;
                    const uint32_t d_tmem = tmem_base + (uint32_t)((acc * p.groups + g) * S::ACC_COLS);
                    if (!wait_bar(smem_u32(&full_bar[stage]), phase, w)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issued = true;
                    // descriptors advance by (byte offset >> 4) in their address field
                    const uint64_t a_desc = desc0 + (uint64_t)((stage * S::STAGE_BYTES) >> 4);
                    const uint64_t b_desc = a_desc + (uint64_t)(S::A_BYTES >> 4);
#pragma unroll
                    for (int j = 0; j < S::KSUB; ++j) {
                        const uint64_t aj = a_desc + (uint64_t)((j * S::A_SUB) >> 4);
                        const uint64_t bj = b_desc + (uint64_t)((j * S::W_SUB) >> 4);
#pragma unroll
                        for (int kk = 0; kk < RT_BK / 16; ++kk) {
                            if constexpr (S::MERGED) {
                                umma_f16_pair(d_tmem, aj + 2 * kk, bj + 2 * kk, IDESC,
                                              (!first || (j | kk) != 0) ? 1u : 0u);
                            } else {   // parts 0 | 1 into blocks 0 | 1, then part 2 added to block 1
                                umma_f16_pair(d_tmem, aj + 2 * kk, bj + 2 * kk, IDESC,
                                              (!first || (j | kk) != 0) ? 1u : 0u);
                                umma_f16_pair(d_tmem + NP, aj + 2 * kk, bj + (uint64_t)((2 * S::P_BYTES) >> 4) + 2 * kk,
                                              IDESC2, 1u);
                            }
                        }
                    }
                    umma_commit_pair(smem_u32(&empty_bar[stage]), 0x3);   // frees the stage in both CTAs
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++kin == p.kb_per_group) {
                        kin = 0;
                        ++g;
                    }
                }
                if (ok) umma_commit_pair(smem_u32(&tfull_bar[acc]), 0x3);
            }
            if (issued) {
                umma_commit_pair(smem_u32(&done_bar), 0x3);
                drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
            }
        } else if (lane == 0 && !leader && first_tile < ntiles) {
            // the peer's TMEM and shared memory are in use until the leader's MMAs end
            drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: one thread per token ----------------
        const int q = warp & 3;
        float psum[S::PER_LANE];   // this warp's sums of p over its tokens, experts [lane NP/32, ...)
#pragma unroll
        for (int j = 0; j < S::PER_LANE; ++j) psum[j] = 0.f;
        const int N = p.N, k = p.k;
        const uint32_t tempty_leader0 = map_to_rank(smem_u32(&tempty_bar[0]), 0);
        const uint32_t tempty_leader1 = map_to_rank(smem_u32(&tempty_bar[1]), 0);
        int it = 0;
        double zacc = 0.0;   // sum over this thread's tokens of log-sum-exp^2
        for (int tile = first_tile; tile < ntiles; tile += tile_step, ++it) {
            const int acc = p.nbuf == 2 ? (it & 1) : 0;
            const uint32_t acc_par = (uint32_t)(p.nbuf == 2 ? ((it >> 1) & 1) : (it & 1));
            const bool got = wait_bar(smem_u32(&tfull_bar[acc]), acc_par, w);
            if (!__all_sync(0xffffffffu, got)) break;   // warp-uniform exit on abort
            tc_fence_after();
            const int64_t t = (int64_t)tile * 2 * RT_BM + (int)rank * RT_BM + q * 32 + lane;
            const bool valid = t < p.T;
            float v[NP];   // logits: the bias, then the partial products in a fixed order
#pragma unroll
            for (int e = 0; e < NP; e += 4) {   // 16-byte broadcast reads
                const float4 b4 = *reinterpret_cast<const float4*>(&s_bias[e]);
                v[e] = b4.x;
                v[e + 1] = b4.y;
                v[e + 2] = b4.z;
                v[e + 3] = b4.w;
            }
            const uint32_t tbase =
                tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.groups * S::ACC_COLS);
            for (int g = 0; g < p.groups; ++g) {   // partial logits of the K groups (and W parts), in order
                constexpr int CH = NP < 64 ? NP : 64;   // columns per TMEM load
#pragma unroll
                for (int part = 0; part < S::BLOCKS; ++part) {
#pragma unroll
                    for (int c = 0; c < NP / CH; ++c) {
                        const uint32_t col = tbase + g * S::ACC_COLS + part * NP + c * CH;
                        uint32_t r[CH];
                        if (CH == 64) tmem_ld64(col, r);
                        else if (CH == 32) tmem_ld32(col, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                        else tmem_ld16(col, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < CH; ++e) v[c * CH + e] += __uint_as_float(r[e]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive_cluster_relaxed(acc ? tempty_leader1 : tempty_leader0);   // the accumulator is free again

            // first choice: the largest logit, lowest index among equals
            const float m = tree_max(v);
            const int i1 = tree_first(v, m);
            // second choice: the largest of the others, lowest index among equals
            float m2 = -INFINITY;
            int i2 = 0;
            if (k == 2) {
                m2 = tree_max(v, i1);
                i2 = tree_first(v, m2, i1);
            }
            // v now holds exp(h - max) = 2^((h - max) log2 e); padding experts
            // hold -inf (their bias), so their terms are 0
            const float m_l2 = m * kLog2e;   // exp(h - max) = 2^(h log2 e - max log2 e), one FMA per expert
#pragma unroll
            for (int e = 0; e < NP; ++e) v[e] = fast_exp2(fmaf(v[e], kLog2e, -m_l2));
            const float s = tree_sum(v);
            const float inv = valid ? 1.f / s : 0.f;
            if (valid) {
                const float lse = m + logf(s);   // log sum_e exp(h_e)
                zacc += (double)lse * (double)lse;
                if (k == 1) {
                    p.idx[t] = i1;
                    p.gate[t] = inv;   // p_{i*} = exp(0) / s
                } else {
                    const float r = fast_exp2((m2 - m) * kLog2e);
                    p.idx[2 * t] = i1;
                    p.idx[2 * t + 1] = i2;
                    p.gate[2 * t] = 1.f / (1.f + r);
                    p.gate[2 * t + 1] = r / (1.f + r);
                }
                if (p.probs) {
#pragma unroll
                    for (int e = 0; e < NP; ++e)
                        if (e < N) p.probs[t * N + e] = v[e] * inv;
                }
                atomicAdd(&s_hist[i1], 1);
            }
#pragma unroll
            for (int e = 0; e < NP; ++e) v[e] *= inv;   // p (0 for a token past T)
            float ts[S::PER_LANE];
            warp_transpose_sum<NP>(v, lane, ts);
#pragma unroll
            for (int j = 0; j < S::PER_LANE; ++j) psum[j] += ts[j];   // tiles in order
        }
#pragma unroll
        for (int j = 0; j < S::PER_LANE; ++j) s_wsum[q][lane * S::PER_LANE + j] = psum[j];
        // ---- this CTA's partials, expert-major: part[e][blockIdx.x] ----
        const int et = tid - 64;   // 0..127 across the four epilogue warps
        s_z[et] = zacc;
        named_bar(1, 128);
        if (et == 0 && p.part_z) {   // fixed order: warp quadrant, then lane
            double zs = 0.0;
            for (int r = 0; r < 128; ++r) zs += s_z[r];
            p.part_z[blockIdx.x] = zs;
        }
        const int Gp = ((int)gridDim.x + 3) & ~3;
        if (et < N) {
            const float ps = (s_wsum[0][et] + s_wsum[1][et]) + (s_wsum[2][et] + s_wsum[3][et]);   // fixed order
            p.part_psum[(int64_t)et * Gp + blockIdx.x] = ps;
            p.part_cnt[(int64_t)et * Gp + blockIdx.x] = s_hist[et];
            __threadfence();
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no CTA leaves while its peer may still signal it
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);

    if (p.defer_aux) return;
    // ---- the last CTA to finish reduces every CTA's partials: f, P, aux ----
    if (tid == 0) s_last = (atomicAdd(p.ticket, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const AuxArgs aa{p.part_cnt, p.part_psum, (int)gridDim.x, p.N, p.T, p.alpha, p.f, p.P, p.aux, p.part_z, p.z};
    aux_reduce_block(aa, reinterpret_cast<double*>(smem));   // pipeline buffers are free now
    if (tid == 0) *p.ticket = 0;                             // ready for the next call
}

// fp32 [N, d] -> bf16 [3, NP, d]: w = w0 + w1 + w2 exactly; rows >= N are zero.
__global__ void split_router_weights_kernel(const float* __restrict__ w_r, int N, int NP, int d,
                                            __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    pdl_launch();
    const int64_t n = (int64_t)NP * d;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(i / d);
        const float wv = e < N ? w_r[i] : 0.f;
        const __nv_bfloat16 w0 = __float2bfloat16_rn(wv);
        const float r1 = wv - __bfloat162float(w0);
        const __nv_bfloat16 w1 = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(w1);
        const __nv_bfloat16 w2 = __float2bfloat16_rn(r2);
        out[i] = w0;
        out[n + i] = w1;
        out[2 * n + i] = w2;
    }
}

template <int NP>
cudaError_t run_router_tc(const RouterArgs& a, cudaStream_t s, int sms) {
    using S = RtShape<NP>;
    cudaError_t err;
    const int threads = 256;
    const int64_t n = (int64_t)NP * a.d;
    const int blocks = (int)((n + threads - 1) / threads < 1024 ? (n + threads - 1) / threads : 1024);
    err = launch_k(split_router_weights_kernel, dim3((unsigned)blocks), dim3(threads), 0, s, 1, a.w_r, a.N, NP, a.d,
                   reinterpret_cast<__nv_bfloat16*>(a.w_split));
    if (err != cudaSuccess) return err;
    CUtensorMap mx, mw;
    if (!make_map_bf16(&mx, a.x, a.T, a.d, RT_BM) || !make_map_bf16(&mw, a.w_split, 3 * NP, a.d, S::W_BOX))
        return cudaErrorInvalidValue;
    RtParams p{};
    const int nkb = (a.d + S::KSUB * RT_BK - 1) / (S::KSUB * RT_BK);   // stages per tile
    // K groups of at most KB_PER_GROUP k-blocks (<= 64 MMAs per full-scale accumulator).
    // Two accumulator buffers (the epilogue overlaps the next tile) when the
    // groups fit in TMEM twice, or when fewer, larger groups of at most 72 MMAs
    // do; otherwise one buffer with groups of <= 64 MMAs.
    int groups = (nkb + S::KB_PER_GROUP - 1) / S::KB_PER_GROUP;
    if (groups < 1) groups = 1;
    const int max2 = S::TMEM_COLS / (2 * S::ACC_COLS);
    int nbuf = 1;
    if (groups <= max2) {
        nbuf = 2;
    } else if (max2 >= 1 && ((nkb + max2 - 1) / max2) * S::MMA_PER_KB <= 72) {
        nbuf = 2;
        groups = max2;
    }
    const int max_groups = S::TMEM_COLS / (nbuf * S::ACC_COLS);
    if (groups > max_groups) groups = max_groups;   // d beyond this bound: more MMAs per accumulator
    p.T = a.T;
    p.N = a.N;
    p.k = a.k;
    p.d = a.d;
    const int kbpg = (nkb + groups - 1) / groups;
    groups = (nkb + kbpg - 1) / kbpg;   // no empty group
    p.nbuf = nbuf;
    p.groups = groups;
    p.kb_per_group = kbpg;
    p.b_r = a.b_r;
    p.idx = a.idx;
    p.gate = a.gate;
    p.probs = a.probs;
    p.part_cnt = a.part_cnt;
    p.part_psum = a.part_psum;
    p.f = a.f;
    p.P = a.P;
    p.aux = a.aux;
    p.alpha = a.alpha;
    p.ticket = a.ticket;
    p.status = a.status;
    p.defer_aux = a.defer_aux ? 1 : 0;
    p.part_z = a.z ? a.part_z : nullptr;
    p.z = a.z;
    p.limit_ns = kWaitLimitNs;
    auto kern = router_tc_kernel<NP>;
    err = once_per_device(reinterpret_cast<const void*>(kern), [](const void* k) {
        return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, RtShape<NP>::SMEM_BYTES);
    });
    if (err != cudaSuccess) return err;
    const int grid = router_tc_grid(a.T, sms);
    return launch_k(kern, dim3((unsigned)grid), dim3(RT_THREADS), S::SMEM_BYTES, s, 2, mx, mw, p);
}

}  // namespace

int router_tc_grid(int64_t T, int sms) {
    const int64_t npairs = (T + 2 * RT_BM - 1) / (2 * RT_BM);
    return 2 * (int)(npairs < sms / 2 ? npairs : sms / 2);
}

// At least 32 padded experts: the pair MMA's N (3 NP merged, NP per part) is
// then a multiple of 32.
int router_tc_padded_experts(int N) { return N <= 32 ? 32 : (N <= 64 ? 64 : 128); }

cudaError_t launch_router_tc(const RouterArgs& a, cudaStream_t s) {
    int sms = 0;
    cudaError_t err = device_sm_count(&sms);
    if (err != cudaSuccess) return err;
    if (a.T == 0)   // no tokens: f, P and the aux loss are zero
        return launch_aux_finalize(a.part_z, a.z, a.part_cnt, a.part_psum, 0, a.N, a.T, a.alpha, a.f, a.P, a.aux, s);
    const int np = router_tc_padded_experts(a.N);
    if (np == 32) return run_router_tc<32>(a, s, sms);
    if (np == 64) return run_router_tc<64>(a, s, sms);
    return run_router_tc<128>(a, s, sms);
}

}  // namespace moe
