// Router of the MoE layer: fp32 logits h = W_r x (+ b_r), softmax, top-k, gate,
// per-block load-balancing partials, and the fp64 aux-loss finalisation.
//
// Definitions: "From Switch Transformer to GLaM", sections "Dense Scaling vs MoE"
// (h(x) = W_r x, p_i = exp(h_i) / sum_j exp(h_j)), "Switch Transformer: making
// MoE simple" (i* = argmax p, gate p_{i*}) and "Load balancing" (f_i, P_i,
// L_aux = alpha N sum f_i P_i); CMU 10-423 Lecture 16, section 2.3 (top-k, then
// softmax over the kept logits; a tie goes to the lower index); "Training
// Stability, Results & Limitations", section 2.1 (the router runs in fp32 on the
// up-cast bf16 input).
//
// Design: the contraction is skinny (N <= 128 outputs per token) and its inputs
// are fp32, so it runs on the FP32 pipe.  A block owns TB tokens and all N
// experts; each thread accumulates TT tokens x TE experts in registers.  The TE
// experts are uniform across a warp, so router weights are read from shared
// memory as broadcasts, while the warp's 32 lanes read 32 consecutive tokens of
// the transposed x tile (conflict-free).  x is read from HBM exactly once.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kDK = 16;   // reduction chunk staged in shared memory

template <int TE, int EG, int kTT>   // kTT: tokens per thread
struct RouterShape {
    static constexpr int TG = 8 / EG;            // token groups (warps per expert group)
    static constexpr int TB = TG * 32 * kTT;     // tokens per block
    static constexpr int NP = TE * EG;           // padded expert count
    static constexpr int XS = kDK * TB;          // x tile floats
    static constexpr int WS = kDK * NP;          // w tile floats
    static constexpr int LG = TB * (NP + 1);     // logits / probabilities
    static constexpr int MAIN = XS + WS;
    static constexpr int SMEM_FLOATS = (MAIN > LG ? MAIN : LG);
};

__device__ __forceinline__ void argmax_merge(float& v, int& i, float ov, int oi) {
    if (ov > v || (ov == v && oi < i)) {
        v = ov;
        i = oi;
    }
}

template <typename XT, int TE, int EG, int kTT>
__global__ void __launch_bounds__(kThreads)
router_kernel(const XT* __restrict__ x, const float* __restrict__ w_r, const float* __restrict__ b_r,
              int64_t T, int d, int N, int k,
              int32_t* __restrict__ idx, float* __restrict__ gate, float* __restrict__ probs,
              int32_t* __restrict__ part_cnt, float* __restrict__ part_psum, double* __restrict__ part_z) {
    using S = RouterShape<TE, EG, kTT>;
    constexpr int VEC = 16 / sizeof(XT);          // elements per 16-byte load
    constexpr int PARTS = kDK / VEC;              // 16-byte loads per row chunk
    constexpr int NL = S::TB * PARTS / kThreads;  // 16-byte loads per thread per chunk
    static_assert(NL >= 1 && (S::TB * PARTS) % kThreads == 0, "loader shape");
    pdl_wait();
    pdl_launch();

    extern __shared__ float smem[];
    float* xs = smem;               // [kDK][TB]
    float* wsm = smem + S::XS;      // [kDK][NP]
    float* lg = smem;               // [TB][NP + 1] after the main loop
    __shared__ int s_cnt[128];
    __shared__ float s_part[kThreads];
    __shared__ double s_zw[kThreads / 32];   // per warp: sum of lse^2 over its tokens

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int eg = warp % EG, tg = warp / EG;
    const int64_t t0 = (int64_t)blockIdx.x * S::TB;
    const int tok_base = tg * 32 * kTT;
    const bool vec_ok = ((size_t)d * sizeof(XT)) % 16 == 0;

    if (tid < 128) s_cnt[tid] = 0;

    float acc[kTT][TE];
#pragma unroll
    for (int i = 0; i < kTT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

    uint4 pre[NL];
    auto load_x = [&](int kc) {
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            int q = tid + kThreads * l;
            int row = q / PARTS, part = q % PARTS;
            int64_t t = t0 + row;
            int col = kc + part * VEC;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t < T) {
                const XT* src = x + t * (int64_t)d + col;
                if (vec_ok && col + VEC <= d) {
                    v = __ldg(reinterpret_cast<const uint4*>(src));
                } else {
                    XT tmp[VEC];
#pragma unroll
                    for (int j = 0; j < VEC; ++j) tmp[j] = (col + j < d) ? src[j] : XT(0.f);
                    v = *reinterpret_cast<uint4*>(tmp);
                }
            }
            pre[l] = v;
        }
    };
    auto store_x = [&]() {
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            int q = tid + kThreads * l;
            int row = q / PARTS, part = q % PARTS;
            const XT* e = reinterpret_cast<const XT*>(&pre[l]);
#pragma unroll
            for (int j = 0; j < VEC; ++j) xs[(part * VEC + j) * S::TB + row] = Elem<XT>::to_f(e[j]);
        }
    };

    load_x(0);
    for (int kc = 0; kc < d; kc += kDK) {
        __syncthreads();   // previous chunk fully consumed
        store_x();
        for (int q = tid; q < kDK * S::NP; q += kThreads) {
            int e = q / kDK, kk = q % kDK;
            float w = 0.f;
            if (e < N && kc + kk < d) w = __ldg(w_r + (int64_t)e * d + kc + kk);
            wsm[kk * S::NP + e] = w;
        }
        __syncthreads();
        if (kc + kDK < d) load_x(kc + kDK);   // overlaps the FMAs below
#pragma unroll
        for (int kk = 0; kk < kDK; ++kk) {
            float xv[kTT];
#pragma unroll
            for (int i = 0; i < kTT; ++i) xv[i] = xs[kk * S::TB + tok_base + lane + 32 * i];
            const float4* wp = reinterpret_cast<const float4*>(wsm + kk * S::NP + eg * TE);
#pragma unroll
            for (int j4 = 0; j4 < TE / 4; ++j4) {
                float4 w = wp[j4];
#pragma unroll
                for (int i = 0; i < kTT; ++i) {
                    acc[i][4 * j4 + 0] = fmaf(xv[i], w.x, acc[i][4 * j4 + 0]);
                    acc[i][4 * j4 + 1] = fmaf(xv[i], w.y, acc[i][4 * j4 + 1]);
                    acc[i][4 * j4 + 2] = fmaf(xv[i], w.z, acc[i][4 * j4 + 2]);
                    acc[i][4 * j4 + 3] = fmaf(xv[i], w.w, acc[i][4 * j4 + 3]);
                }
            }
        }
    }
    __syncthreads();   // x/w tiles are dead; the logits reuse the space

    // ---- logits -> shared memory ------------------------------------------------
#pragma unroll
    for (int i = 0; i < kTT; ++i) {
        int tok = tok_base + lane + 32 * i;
#pragma unroll
        for (int j = 0; j < TE; ++j) {
            int e = eg * TE + j;
            float v = acc[i][j];
            if (e < N && b_r) v += __ldg(b_r + e);
            lg[tok * (S::NP + 1) + e] = v;
        }
    }
    __syncthreads();

    // ---- per token: softmax, top-k, gate ----------------------------------------
    constexpr int MPL = (S::NP + 31) / 32;
    const int64_t rem_t = T - t0;
    const int tb_valid = rem_t < (int64_t)S::TB ? (int)rem_t : S::TB;
    double zacc = 0.0;   // sum over this warp's (thread's) tokens of log-sum-exp^2
    if (S::NP <= 32) {
        // few experts: one thread per token, its logits in registers (no
        // shuffle chains; the same arithmetic and order per token as below)
        for (int tok = tid; tok < tb_valid; tok += kThreads) {
            float* row = lg + tok * (S::NP + 1);
            float v[S::NP];
            float m = -INFINITY;
#pragma unroll
            for (int e = 0; e < S::NP; ++e) {
                v[e] = e < N ? row[e] : -INFINITY;
                m = fmaxf(m, v[e]);
            }
            float ex[S::NP];
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < S::NP; ++e) {
                ex[e] = e < N ? expf(v[e] - m) : 0.f;
                s += ex[e];
            }
            float bv = -INFINITY, cv = -INFINITY;
            int bi = 0x7fffffff, ci = 0x7fffffff;
#pragma unroll
            for (int e = 0; e < S::NP; ++e)
                if (e < N) argmax_merge(bv, bi, v[e], e);
            if (k == 2) {
#pragma unroll
                for (int e = 0; e < S::NP; ++e)
                    if (e < N && e != bi) argmax_merge(cv, ci, v[e], e);
            }
            const float inv = 1.f / s;
            const int64_t t = t0 + tok;
#pragma unroll
            for (int e = 0; e < S::NP; ++e) {
                if (e < N) {
                    const float pe = ex[e] * inv;
                    row[e] = pe;
                    if (probs) probs[t * N + e] = pe;
                }
            }
            const float lse = m + logf(s);
            zacc += (double)lse * (double)lse;
            atomicAdd(&s_cnt[bi], 1);
            if (k == 1) {
                idx[t] = bi;
                gate[t] = inv;
            } else {
                const float r = expf(cv - bv);
                idx[2 * t] = bi;
                idx[2 * t + 1] = ci;
                gate[2 * t] = 1.f / (1.f + r);
                gate[2 * t + 1] = r / (1.f + r);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zacc += __shfl_xor_sync(0xffffffffu, zacc, o);
    }
    for (int tok = warp; S::NP > 32 && tok < tb_valid; tok += kThreads / 32) {
        float* row = lg + tok * (S::NP + 1);
        float v[MPL];
        float m = -INFINITY;
#pragma unroll
        for (int q = 0; q < MPL; ++q) {
            int e = lane + 32 * q;
            v[q] = (e < N) ? row[e] : -INFINITY;
            m = fmaxf(m, v[q]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float ex[MPL];
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < MPL; ++q) {
            ex[q] = (lane + 32 * q < N) ? expf(v[q] - m) : 0.f;
            s += ex[q];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        // first choice: largest logit, lower index on ties
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < MPL; ++q) {
            int e = lane + 32 * q;
            if (e < N) argmax_merge(bv, bi, v[q], e);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            argmax_merge(bv, bi, ov, oi);
        }
        int i2 = 0;
        float v2 = 0.f;
        if (k == 2) {
            float cv = -INFINITY;
            int ci = 0x7fffffff;
#pragma unroll
            for (int q = 0; q < MPL; ++q) {
                int e = lane + 32 * q;
                if (e < N && e != bi) argmax_merge(cv, ci, v[q], e);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, cv, o);
                int oi = __shfl_xor_sync(0xffffffffu, ci, o);
                argmax_merge(cv, ci, ov, oi);
            }
            i2 = ci;
            v2 = cv;
        }
        const float inv = 1.f / s;
        const int64_t t = t0 + tok;
#pragma unroll
        for (int q = 0; q < MPL; ++q) {
            int e = lane + 32 * q;
            if (e < N) {
                float p = ex[q] * inv;
                row[e] = p;
                if (probs) probs[t * N + e] = p;
            }
        }
        if (lane == 0) {
            const float lse = m + logf(s);   // log sum_e exp(h_e)
            zacc += (double)lse * (double)lse;
            atomicAdd(&s_cnt[bi], 1);
            if (k == 1) {
                idx[t] = bi;
                gate[t] = inv;   // p_{i*} = exp(h_{i*} - max) / s = 1 / s
            } else {
                float r = expf(v2 - bv);
                idx[2 * t] = bi;
                idx[2 * t + 1] = i2;
                gate[2 * t] = 1.f / (1.f + r);
                gate[2 * t + 1] = r / (1.f + r);
            }
        }
    }
    if (lane == 0) s_zw[warp] = zacc;
    __syncthreads();
    if (part_z && tid == 0) {
        double zs = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) zs += s_zw[w];
        part_z[blockIdx.x] = zs;
    }

    // ---- block partials in a fixed order: sum_t p[t][e], count of top-1 == e ----
    int npow = 8;
    while (npow < N) npow <<= 1;
    const int ns = kThreads / npow;            // token slices
    const int len = (S::TB + ns - 1) / ns;
    {
        int e = tid % npow, sl = tid / npow;
        float acc_p = 0.f;
        if (e < N) {
            int lo = sl * len, hi = min(lo + len, tb_valid);
            for (int tok = lo; tok < hi; ++tok) acc_p += lg[tok * (S::NP + 1) + e];
        }
        s_part[tid] = acc_p;
    }
    __syncthreads();
    if (tid < N) {
        float acc_p = 0.f;
        for (int sl = 0; sl < ns; ++sl) acc_p += s_part[sl * npow + tid];
        part_psum[(int64_t)blockIdx.x * N + tid] = acc_p;
        part_cnt[(int64_t)blockIdx.x * N + tid] = s_cnt[tid];
    }
}

// f_i, P_i, aux from the per-block partials; fp64, fixed reduction order.
__global__ void __launch_bounds__(1024)
aux_finalize_kernel(const double* __restrict__ part_z, double* __restrict__ z,
                    const int32_t* __restrict__ part_cnt, const float* __restrict__ part_psum,
                    int nblk, int N, int64_t T, float alpha,
                    double* __restrict__ f, double* __restrict__ P, double* __restrict__ aux) {
    __shared__ double sp[1024];
    __shared__ double sc[1024];
    __shared__ double sfp[128];
    pdl_wait();
    pdl_launch();
    int npow = 1;
    while (npow < N) npow <<= 1;
    const int tpe = 1024 / npow;
    const int tid = threadIdx.x, e = tid % npow, j = tid / npow;
    double a = 0.0, c = 0.0;
    if (e < N) {   // blocks j, j + tpe, ... in order, 8 independent loads in flight
        for (int b0 = j; b0 < nblk; b0 += 8 * tpe) {
            float pv[8];
            int cv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int b = b0 + u * tpe;
                pv[u] = b < nblk ? part_psum[(int64_t)b * N + e] : 0.f;
                cv[u] = b < nblk ? part_cnt[(int64_t)b * N + e] : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (b0 + u * tpe < nblk) {
                    a += (double)pv[u];
                    c += (double)cv[u];
                }
            }
        }
    }
    sp[tid] = a;
    sc[tid] = c;
    __syncthreads();
    if (tid < N) {
        double pa = 0.0, ca = 0.0;
        for (int q = 0; q < tpe; ++q) {
            pa += sp[q * npow + tid];
            ca += sc[q * npow + tid];
        }
        double Pe = T > 0 ? pa / (double)T : 0.0;
        double fe = T > 0 ? ca / (double)T : 0.0;
        if (P) P[tid] = Pe;
        if (f) f[tid] = fe;
        sfp[tid] = fe * Pe;
    }
    __syncthreads();
    if (tid == 0 && aux) {
        double s = 0.0;
        for (int q = 0; q < N; ++q) s += sfp[q];
        *aux = (double)alpha * (double)N * s;
    }
    if (z && tid < 32) z_reduce_warp(part_z, nblk, T, z);
}

template <typename XT, int TE, int EG, int kTT>
cudaError_t launch_router_t(const RouterArgs& a, cudaStream_t s) {
    using S = RouterShape<TE, EG, kTT>;
    const int nblk = (int)((a.T + S::TB - 1) / S::TB);
    const size_t smem = sizeof(float) * S::SMEM_FLOATS;
    auto kern = router_kernel<XT, TE, EG, kTT>;
    cudaError_t err = once_per_device(reinterpret_cast<const void*>(kern), [](const void* k) {
        return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)(sizeof(float) * RouterShape<TE, EG, kTT>::SMEM_FLOATS));
    });
    if (err != cudaSuccess) return err;
    if (nblk > 0) {
        err = launch_k(kern, dim3((unsigned)nblk), dim3(kThreads), smem, s, 1, reinterpret_cast<const XT*>(a.x), a.w_r,
                       a.b_r, a.T, a.d, a.N, a.k, a.idx, a.gate, a.probs, a.part_cnt, a.part_psum,
                       a.z ? a.part_z : nullptr);
        if (err != cudaSuccess) return err;
    }
    return launch_aux_finalize(a.part_z, a.z, a.part_cnt, a.part_psum, nblk, a.N, a.T, a.alpha, a.f, a.P, a.aux, s);
}

// Few tokens (fewer than 64 blocks of the four-tokens-per-thread shape): one
// token per thread and 64- or 128-token blocks, so the work spreads over more
// SMs (the 512-token fp32 layer: 4 blocks instead of 1).
bool small_batch(int64_t T, int N) {
    const int64_t tb = N <= 8 ? RouterShape<8, 1, 4>::TB : RouterShape<16, 1, 4>::TB;
    return (T + tb - 1) / tb < 64;
}

template <typename XT>
cudaError_t launch_router_x(const RouterArgs& a, cudaStream_t s) {
    if (small_batch(a.T, a.N)) {
        if (a.N <= 8) return launch_router_t<XT, 4, 2, 1>(a, s);
        if (a.N <= 16) return launch_router_t<XT, 4, 4, 1>(a, s);
        if (a.N <= 32) return launch_router_t<XT, 8, 4, 1>(a, s);
    }
    if (a.N <= 8) return launch_router_t<XT, 8, 1, 4>(a, s);
    if (a.N <= 16) return launch_router_t<XT, 16, 1, 4>(a, s);
    if (a.N <= 32) return launch_router_t<XT, 16, 2, 4>(a, s);
    if (a.N <= 64) return launch_router_t<XT, 16, 4, 4>(a, s);
    return launch_router_t<XT, 16, 8, 4>(a, s);
}

}  // namespace

int router_blocks(int64_t T, int N) {
    int tb;
    if (small_batch(T, N) && N <= 32) tb = N <= 8 ? RouterShape<4, 2, 1>::TB : (N <= 16 ? RouterShape<4, 4, 1>::TB : RouterShape<8, 4, 1>::TB);
    else if (N <= 8) tb = RouterShape<8, 1, 4>::TB;
    else if (N <= 16) tb = RouterShape<16, 1, 4>::TB;
    else if (N <= 32) tb = RouterShape<16, 2, 4>::TB;
    else if (N <= 64) tb = RouterShape<16, 4, 4>::TB;
    else tb = RouterShape<16, 8, 4>::TB;
    return (int)((T + tb - 1) / tb);
}

int router_partial_rows(int64_t T, int N) {
    const int tc_rows = (int)((2 * ((T + 255) / 256) + 3) / 4 * 4);   // >= the tensor-core router's grid, rounded to 4
    const int simt_rows = router_blocks(T, N);
    return tc_rows > simt_rows ? tc_rows : simt_rows;
}

cudaError_t launch_aux_finalize(const double* part_z, double* z, const int32_t* part_cnt, const float* part_psum,
                                int nblk, int N, int64_t T, float alpha, double* f, double* P, double* aux,
                                cudaStream_t s) {
    return launch_k(aux_finalize_kernel, dim3(1), dim3(1024), 0, s, 1, part_z, z, part_cnt, part_psum, nblk, N, T,
                    alpha, f, P, aux);
}

// bf16 activations: the tensor-core router (exact three-way split of W_r);
// fp32 activations: the FP32-pipe router.
cudaError_t launch_router(const RouterArgs& a, cudaStream_t s) {
    if (a.dtype == MOE_BF16) return launch_router_tc(a, s);
    return launch_router_x<float>(a, s);
}

}  // namespace moe
