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
// is the fp32 dot product up to accumulation rounding -- three bf16 MMAs per
// K step.  The tensor core's fp32 accumulation truncates, so its error grows
// with the number of MMAs summed into one accumulator; the K loop is therefore
// cut into G groups of at most 8 k-blocks (<= 96 MMAs), each accumulating into
// its own TMEM column block, and the epilogue adds the G partial logits in fp32
// with round-to-nearest in a fixed order.  The router then costs about one read
// of x from HBM instead of 2 d N FP32-pipe FLOPs per token.
//
// Kernel: persistent, 192 threads: warp 0 TMA producer (x tile 128 x 64 and
// the three W parts, NP x 64 each, 128-byte swizzle), warp 1 TMEM allocator +
// MMA issuer (M = 128 tokens, N = NP padded experts, K = 16), warps 2-5
// epilogue with one thread per token: the thread holds its token's NP logits
// (tcgen05.ld), computes max, softmax, top-1/top-2 and the gate in registers,
// and writes idx/gate (and probs).  Per-tile partial sums of p and top-1
// counts are reduced in a fixed order (lanes in a warp through shared memory,
// then the four warps in quadrant order), so the aux loss is deterministic.
#include "tc_common.cuh"

namespace moe {
using namespace tc;
namespace {

constexpr int RT_THREADS = 192;
constexpr int RT_BM = 128;
constexpr int RT_BK = 64;

template <int NP>
struct RtShape {
    static constexpr int A_BYTES = RT_BM * RT_BK * 2;
    static constexpr int P_BYTES = NP * RT_BK * 2;             // one W part
    static constexpr int STAGE_BYTES = A_BYTES + 3 * P_BYTES;
    static constexpr int STAGES = NP <= 64 ? 4 : 3;
    static constexpr int RED_FLOATS = 4 * 32 * 33;              // per-warp transpose buffers
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + RED_FLOATS * 4;
    static constexpr int TMEM_COLS = 512;                      // 2 buffers x G groups x NP columns
    static constexpr int MAX_GROUPS = TMEM_COLS / (2 * NP);
};
constexpr int RT_KB_PER_GROUP = 8;

struct RtParams {
    int64_t T;
    int N, k, d;
    int groups;   // K groups with separate accumulators
    int kb_per_group;
    const float* b_r;
    int32_t* idx;
    float* gate;
    float* probs;
    int32_t* part_cnt;
    float* part_psum;
    int32_t* status;
    long long limit_ns;
};

__device__ __forceinline__ void take_max(float& v, int& i, float ov, int oi) {
    if (ov > v || (ov == v && oi < i)) {
        v = ov;
        i = oi;
    }
}

template <int NP>
__global__ void __launch_bounds__(RT_THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, const RtParams p) {
    using S = RtShape<NP>;
    constexpr uint32_t IDESC = idesc_bf16_f32(RT_BM, NP);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    float* red = reinterpret_cast<float*>(smem + S::STAGES * S::STAGE_BYTES);
    __shared__ __align__(8) uint64_t full_bar[S::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[S::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_wpart[4][NP];
    __shared__ int s_hist[NP];
    __shared__ int s_ok[2][4];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull_bar[a]), 1);
            mbar_init(smem_u32(&tempty_bar[a]), 128);
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
    if (warp == 1) tmem_alloc(&s_tmem, S::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = s_tmem;
    const int ntiles = (int)((p.T + RT_BM - 1) / RT_BM);
    const int nkb = (p.d + RT_BK - 1) / RT_BK;
    const Waiter w{&s_abort, p.status, p.limit_ns};

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int last_par[S::STAGES];
#pragma unroll
            for (int s = 0; s < S::STAGES; ++s) last_par[s] = -1;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(smem_u32(&empty_bar[stage]), phase ^ 1u, w)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t a_dst = smem_u32(smem + stage * S::STAGE_BYTES);
                    mbar_expect_tx(fb, S::STAGE_BYTES);
                    tma_load_2d(a_dst, &tmX, fb, kb * RT_BK, tile * RT_BM);
#pragma unroll
                    for (int part = 0; part < 3; ++part)
                        tma_load_2d(a_dst + S::A_BYTES + part * S::P_BYTES, &tmW, fb, kb * RT_BK, part * NP);
                    last_par[stage] = (int)phase;
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < S::STAGES; ++s)
                if (last_par[s] >= 0) drain_bar(smem_u32(&full_bar[s]), (uint32_t)last_par[s], p.limit_ns, p.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
                if (!wait_bar(smem_u32(&tempty_bar[acc]), acc_par ^ 1u, w)) break;
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb) {
                    const int g = kb / p.kb_per_group;
                    const bool first = kb == g * p.kb_per_group;
                    const uint32_t d_tmem = tmem_base + (uint32_t)((acc * p.groups + g) * NP);
                    if (!wait_bar(smem_u32(&full_bar[stage]), phase, w)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issued = true;
                    const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < RT_BK / 16; ++kk) {
#pragma unroll
                        for (int part = 0; part < 3; ++part) {
                            const uint32_t b_addr = a_addr + S::A_BYTES + part * S::P_BYTES;
                            umma_f16(d_tmem, umma_desc(a_addr + kk * 32), umma_desc(b_addr + kk * 32), IDESC,
                                     (!first || (kk | part) != 0) ? 1u : 0u);
                        }
                    }
                    umma_commit(smem_u32(&empty_bar[stage]));
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit(smem_u32(&tfull_bar[acc]));
            }
            if (issued) {
                umma_commit(smem_u32(&done_bar));
                drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: one thread per token ----------------
        const int q = warp & 3;
        float* tr = red + q * 32 * 33;   // this warp's 32 x 33 transpose buffer
        const int N = p.N, k = p.k;
        int it = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
            // all four epilogue warps agree before going on, so that none is left
            // waiting at the named barriers below if another gave up
            const bool got = __all_sync(0xffffffffu, wait_bar(smem_u32(&tfull_bar[acc]), acc_par, w));
            if (lane == 0) s_ok[it & 1][q] = got ? 1 : 0;
            named_bar(1, 128);
            if (!(s_ok[it & 1][0] & s_ok[it & 1][1] & s_ok[it & 1][2] & s_ok[it & 1][3])) break;
            tc_fence_after();
            const int64_t t = (int64_t)tile * RT_BM + q * 32 + lane;
            const bool valid = t < p.T;
            float v[NP];
#pragma unroll
            for (int e = 0; e < NP; ++e) v[e] = 0.f;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.groups * NP);
            for (int g = 0; g < p.groups; ++g) {   // partial logits of the K groups, in order
#pragma unroll
                for (int c = 0; c < NP / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tbase + g * NP + c * 16, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[c * 16 + j] += __uint_as_float(r[j]);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty_bar[acc]));   // the accumulator is free again

            float m = -INFINITY;
            int i1 = 0x7fffffff;
#pragma unroll
            for (int e = 0; e < NP; ++e) {
                if (e < N) {
                    if (p.b_r) v[e] += __ldg(p.b_r + e);
                    take_max(m, i1, v[e], e);
                }
            }
            // second choice: largest logit among the others (lower index on ties)
            float m2 = -INFINITY;
            int i2 = 0x7fffffff;
            if (k == 2) {
#pragma unroll
                for (int e = 0; e < NP; ++e)
                    if (e < N && e != i1) take_max(m2, i2, v[e], e);
            }
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < NP; ++e) {
                float ex = (e < N) ? expf(v[e] - m) : 0.f;
                s += ex;
                v[e] = ex;   // v now holds exp(h - max)
            }
            const float inv = 1.f / s;
            if (valid) {
                if (k == 1) {
                    p.idx[t] = i1;
                    p.gate[t] = inv;   // p_{i*} = exp(0) / s
                } else {
                    const float r = expf(m2 - m);
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
            // per-tile sums of p over the tile's tokens: lanes (tokens) in order
            // inside a warp through a 32 x 33 transpose, then warps 0..3
#pragma unroll
            for (int c = 0; c < NP / 32 + (NP % 32 ? 1 : 0); ++c) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int e = c * 32 + j;
                    if (e < NP) tr[lane * 33 + j] = (valid && e < N) ? v[e] * inv : 0.f;
                }
                __syncwarp();
                float a = 0.f;
                for (int l = 0; l < 32; ++l) a += tr[l * 33 + lane];
                if (c * 32 + lane < NP) s_wpart[q][c * 32 + lane] = a;
                __syncwarp();
            }
            named_bar(1, 128);
            const int et = tid - 64;   // 0..127 across the four epilogue warps
            if (et < N) {
                const float ps = ((s_wpart[0][et] + s_wpart[1][et]) + s_wpart[2][et]) + s_wpart[3][et];
                p.part_psum[(int64_t)tile * N + et] = ps;
                p.part_cnt[(int64_t)tile * N + et] = s_hist[et];
                s_hist[et] = 0;
            }
            named_bar(1, 128);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, S::TMEM_COLS);
}

// fp32 [N, d] -> bf16 [3, NP, d]: w = w0 + w1 + w2 exactly; rows >= N are zero.
__global__ void split_router_weights_kernel(const float* __restrict__ w_r, int N, int NP, int d,
                                            __nv_bfloat16* __restrict__ out) {
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
    split_router_weights_kernel<<<blocks, threads, 0, s>>>(a.w_r, a.N, NP, a.d,
                                                           reinterpret_cast<__nv_bfloat16*>(a.w_split));
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    CUtensorMap mx, mw;
    if (!make_map_bf16(&mx, a.x, a.T, a.d, RT_BM) || !make_map_bf16(&mw, a.w_split, 3 * NP, a.d, NP))
        return cudaErrorInvalidValue;
    RtParams p{};
    const int nkb = (a.d + RT_BK - 1) / RT_BK;
    int groups = (nkb + RT_KB_PER_GROUP - 1) / RT_KB_PER_GROUP;
    if (groups > S::MAX_GROUPS) groups = S::MAX_GROUPS;
    p.T = a.T;
    p.N = a.N;
    p.k = a.k;
    p.d = a.d;
    if (groups < 1) groups = 1;
    const int kbpg = (nkb + groups - 1) / groups;
    groups = (nkb + kbpg - 1) / kbpg;   // no empty group
    p.groups = groups;
    p.kb_per_group = kbpg;
    p.b_r = a.b_r;
    p.idx = a.idx;
    p.gate = a.gate;
    p.probs = a.probs;
    p.part_cnt = a.part_cnt;
    p.part_psum = a.part_psum;
    p.status = a.status;
    p.limit_ns = kWaitLimitNs;
    auto kern = router_tc_kernel<NP>;
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES)) != cudaSuccess)
        return err;
    const int ntiles = (int)((a.T + RT_BM - 1) / RT_BM);
    const int grid = ntiles < sms ? ntiles : sms;
    kern<<<grid, RT_THREADS, S::SMEM_BYTES, s>>>(mx, mw, p);
    return cudaGetLastError();
}

}  // namespace

int router_tc_padded_experts(int N) { return N <= 16 ? 16 : (N <= 32 ? 32 : (N <= 64 ? 64 : 128)); }

cudaError_t launch_router_tc(const RouterArgs& a, cudaStream_t s) {
    int dev = 0, sms = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    if (a.T > 0) {
        const int np = router_tc_padded_experts(a.N);
        if (np == 16) err = run_router_tc<16>(a, s, sms);
        else if (np == 32) err = run_router_tc<32>(a, s, sms);
        else if (np == 64) err = run_router_tc<64>(a, s, sms);
        else err = run_router_tc<128>(a, s, sms);
        if (err != cudaSuccess) return err;
    }
    return launch_aux_finalize(a.part_cnt, a.part_psum, (int)((a.T + RT_BM - 1) / RT_BM), a.N, a.T, a.alpha, a.f,
                               a.P, a.aux, s);
}

}  // namespace moe
