// Router backward on the FP32 pipe: gradients of sum_{t,r} dgate[t,r] g_{t,r}
// + L_aux with respect to the router logits h, W_r, b_r and the router input x.
//
//  - gate path ("From Switch Transformer to GLaM": y = p_{i*} E_{i*}(x) for
//    top-1, y = w1 E_{i1} + w2 E_{i2} with w the softmax over the two kept
//    logits for top-2; the expert choice itself carries no gradient):
//      top-1: dh_j += dgate p_{i*} (delta_{j i*} - p_j);
//      top-2: dh_{i1} += (dg1 - dg2) g1 g2, dh_{i2} -= (dg1 - dg2) g1 g2.
//  - load-balancing loss (CMU 10-423 Lecture 16, section 4.2: f_i is counted
//    and carries no gradient, P_i = mean_t p_{t,i} carries coefficient f_i):
//      dh_j += p_j (a_j - sum_i p_i a_i), a_i = alpha N f_i / T.
//  - dW_r = dh^T x, db_r = sum_t dh_t (a contraction over tokens: per
//    512-token chunk partials, then a fixed-order fp64 sum over chunks), and
//    dx_t = dh_t W_r.
// Kernels: router_bwd_dh_kernel (a warp per eight tokens); for bf16 x the two
// contractions run on the tensor cores through exact three-way bf16 splits
// (rbwd_* kernels, the grouped GEMMs of gemm_bwd.cu); for fp32 x on the FP32
// pipe: router_bwd_dw_kernel (32 experts x 128 columns per block over one
// token chunk), router_bwd_reduce_kernel, router_bwd_dx_kernel (64 tokens x
// 128 columns).  All sums run in a fixed order: results are bit-identical run
// to run.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kBwdChunk = 512;   // tokens per dW_r partial

// dL/dh of kDhTokens consecutive tokens per warp (lane: experts lane + 32 q):
// the load-balancing coefficients a_e are formed once per warp, and every
// token's probabilities are loaded before the first is used (with a warp per
// token, 8192 blocks each living about a microsecond bounded the kernel).
constexpr int kDhTokens = 8;

__global__ void __launch_bounds__(256)
router_bwd_dh_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx, const float* __restrict__ gate,
                     const float* __restrict__ dgate, const double* __restrict__ f, float alpha, int64_t T, int N,
                     int k, float* __restrict__ dh) {
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t t0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * kDhTokens;
    if (t0 >= T) return;
    float av[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        av[q] = e < N ? (float)((double)alpha * (double)N * f[e] / (double)T) : 0.f;
    }
    float pv[kDhTokens][4];
#pragma unroll
    for (int i = 0; i < kDhTokens; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = lane + 32 * q;
            pv[i][q] = (t0 + i < T && e < N) ? probs[(t0 + i) * N + e] : 0.f;
        }
#pragma unroll
    for (int i = 0; i < kDhTokens; ++i) {
        const int64_t t = t0 + i;
        if (t >= T) break;   // warp-uniform
        float spa = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) spa = fmaf(pv[i][q], av[q], spa);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) spa += __shfl_xor_sync(0xffffffffu, spa, o);
        float gv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) gv[q] = pv[i][q] * (av[q] - spa);
        if (k == 1) {
            const int is = idx[t];
            const float c = dgate[t] * gate[t];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = lane + 32 * q;
                gv[q] += c * ((e == is ? 1.f : 0.f) - pv[i][q]);
            }
        } else {
            const int i1 = idx[2 * t], i2 = idx[2 * t + 1];
            const float g1 = gate[2 * t], g2 = gate[2 * t + 1];
            const float c = (dgate[2 * t] - dgate[2 * t + 1]) * g1 * g2;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = lane + 32 * q;
                if (e == i1) gv[q] += c;
                if (e == i2) gv[q] -= c;
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = lane + 32 * q;
            if (e < N) dh[t * N + e] = gv[q];
        }
    }
}

// part_dw[chunk][n][c] = sum over the chunk's tokens of dh[t][n] x[t][c];
// blocks with blockIdx.z == 0 also write part_db[chunk][n].
template <typename XT>
__global__ void __launch_bounds__(256)
router_bwd_dw_kernel(const float* __restrict__ dh, const XT* __restrict__ x, int64_t T, int N, int d,
                     float* __restrict__ part_dw, float* __restrict__ part_db) {
    pdl_wait();
    pdl_launch();
    __shared__ float s_dh[32][33];    // [token][expert]
    __shared__ float s_x[32][132];    // [token][column]
    const int tid = threadIdx.x;
    const int chunk = blockIdx.x, n0 = blockIdx.y * 32, c0 = blockIdx.z * 128;
    const int64_t t_lo = (int64_t)chunk * kBwdChunk;
    const int64_t t_hi = t_lo + kBwdChunk < T ? t_lo + kBwdChunk : T;
    const int tn = tid >> 5, tc = tid & 31;   // thread: experts 4 tn .. 4 tn + 3, columns tc + 32 j
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    float dbacc = 0.f;   // thread tid < 32: expert n0 + tid
    for (int64_t t0 = t_lo; t0 < t_hi; t0 += 32) {
        for (int q = tid; q < 32 * 32; q += 256) {
            const int r = q >> 5, c = q & 31;
            const int64_t t = t0 + r;
            s_dh[r][c] = (t < t_hi && n0 + c < N) ? dh[t * N + n0 + c] : 0.f;
        }
        for (int q = tid; q < 32 * 128; q += 256) {
            const int r = q >> 7, c = q & 127;
            const int64_t t = t0 + r;
            s_x[r][c] = (t < t_hi && c0 + c < d) ? Elem<XT>::to_f(x[t * d + c0 + c]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = s_dh[r][4 * tn + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = s_x[r][tc + 32 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (blockIdx.z == 0 && tid < 32)
            for (int r = 0; r < 32; ++r) dbacc += s_dh[r][tid];
        __syncthreads();
    }
    float* pw = part_dw + (int64_t)chunk * N * d;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = n0 + 4 * tn + i;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + tc + 32 * j;
            if (c < d) pw[(int64_t)n * d + c] = acc[i][j];
        }
    }
    if (blockIdx.z == 0 && tid < 32 && n0 + tid < N) part_db[(int64_t)chunk * N + n0 + tid] = dbacc;
}

// dw[n][c] = sum over chunks, in order, of the partials (fp64 accumulation)
__global__ void __launch_bounds__(256)
router_bwd_reduce_kernel(const float* __restrict__ part_dw, const float* __restrict__ part_db, int nchunk, int N,
                         int d, float* __restrict__ dw, float* __restrict__ db) {
    pdl_wait();
    pdl_launch();
    const int64_t nd = (int64_t)N * d;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nd + N; i += (int64_t)gridDim.x * blockDim.x) {
        double acc = 0.0;
        if (i < nd) {
            for (int c = 0; c < nchunk; ++c) acc += (double)part_dw[(int64_t)c * nd + i];
            if (dw) dw[i] = (float)acc;
        } else {
            const int64_t n = i - nd;
            for (int c = 0; c < nchunk; ++c) acc += (double)part_db[(int64_t)c * N + n];
            if (db) db[n] = (float)acc;
        }
    }
}

// dx[t][c] = sum_n dh[t][n] W_r[n][c]
__global__ void __launch_bounds__(256)
router_bwd_dx_kernel(const float* __restrict__ dh, const float* __restrict__ w_r, int64_t T, int N, int d,
                     float* __restrict__ dx) {
    pdl_wait();
    pdl_launch();
    __shared__ float s_dh[64][33];   // [token][expert]
    __shared__ float s_w[32][132];   // [expert][column]
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * 64;
    const int c0 = blockIdx.y * 128;
    const int tt = tid >> 5, tc = tid & 31;   // thread: tokens 8 tt .. 8 tt + 7, columns tc + 32 j
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int n0 = 0; n0 < N; n0 += 32) {
        for (int q = tid; q < 64 * 32; q += 256) {
            const int r = q >> 5, c = q & 31;
            const int64_t t = t0 + r;
            s_dh[r][c] = (t < T && n0 + c < N) ? dh[t * N + n0 + c] : 0.f;
        }
        for (int q = tid; q < 32 * 128; q += 256) {
            const int r = q >> 7, c = q & 127;
            s_w[r][c] = (n0 + r < N && c0 + c < d) ? w_r[(int64_t)(n0 + r) * d + c0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int n = 0; n < 32; ++n) {
            float b[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = s_w[n][tc + 32 * j];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a = s_dh[8 * tt + i][n];
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a, b[j], acc[i][j]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t t = t0 + 8 * tt + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + tc + 32 * j;
            if (c < d) dx[t * d + c] = acc[i][j];
        }
    }
}

// ---- tensor-core contractions (bf16 x) ---------------------------------------
// x is exact in bf16; dh and W_r (fp32) split exactly into three bf16 parts
// each (v = v0 + v1 + v2).  dW_r = sum_j dh_j^T x (three exact products, fp32
// accumulation per token chunk, fp64 over chunks and parts); dx = dh W_r from
// the six part products dh_i w_j with i + j <= 2 (the dropped ones are below
// 2^-24 of the result), one GEMM with K = 6 NP16 over
// [dh0 dh0 dh1 dh0 dh1 dh2] x [w0; w1; w0; w2; w1; w0].
__device__ __forceinline__ void split3(float v, __nv_bfloat16& a, __nv_bfloat16& b, __nv_bfloat16& c) {
    a = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(a);
    b = __float2bfloat16_rn(r1);
    c = __float2bfloat16_rn(r1 - __bfloat162float(b));
}

// A thread splits eight consecutive experts of one token (NP16 is a multiple
// of 16), so every row segment it writes is one 16-byte store.
__global__ void __launch_bounds__(256)
rbwd_split_kernel(const float* __restrict__ dh, int64_t T, int N, int NP16, __nv_bfloat16* __restrict__ adx,
                  __nv_bfloat16* __restrict__ adw, int32_t* __restrict__ offs, int64_t chunk, int nchunk) {
    pdl_wait();
    pdl_launch();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        offs[0] = 0;
        offs[1] = (int32_t)T;
        for (int i = 0; i <= nchunk; ++i) offs[2 + i] = (int32_t)min((int64_t)i * chunk, T);
    }
    const int per_row = NP16 / 8;
    const int64_t n_el = T * per_row;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < n_el; q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = q / per_row;
        const int e0 = (int)(q - t * per_row) * 8;
        uint32_t p0[4], p1[4], p2[4];   // the eight experts' three parts, packed bf16 pairs
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            __nv_bfloat16 a0, a1, a2, b0, b1, b2;
            const int e = e0 + 2 * h;
            split3(e < N ? dh[t * N + e] : 0.f, a0, a1, a2);
            split3(e + 1 < N ? dh[t * N + e + 1] : 0.f, b0, b1, b2);
            p0[h] = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(b0) << 16);
            p1[h] = (uint32_t)__bfloat16_as_ushort(a1) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
            p2[h] = (uint32_t)__bfloat16_as_ushort(a2) | ((uint32_t)__bfloat16_as_ushort(b2) << 16);
        }
        const uint4 v0 = make_uint4(p0[0], p0[1], p0[2], p0[3]);
        const uint4 v1 = make_uint4(p1[0], p1[1], p1[2], p1[3]);
        const uint4 v2 = make_uint4(p2[0], p2[1], p2[2], p2[3]);
        __nv_bfloat16* rx = adx + t * (6 * NP16) + e0;   // K segments: parts 0, 0, 1, 0, 1, 2
        *reinterpret_cast<uint4*>(rx) = v0;
        *reinterpret_cast<uint4*>(rx + NP16) = v0;
        *reinterpret_cast<uint4*>(rx + 2 * NP16) = v1;
        *reinterpret_cast<uint4*>(rx + 3 * NP16) = v0;
        *reinterpret_cast<uint4*>(rx + 4 * NP16) = v1;
        *reinterpret_cast<uint4*>(rx + 5 * NP16) = v2;
        __nv_bfloat16* rw = adw + t * (3 * NP16) + e0;
        *reinterpret_cast<uint4*>(rw) = v0;
        *reinterpret_cast<uint4*>(rw + NP16) = v1;
        *reinterpret_cast<uint4*>(rw + 2 * NP16) = v2;
    }
}

__global__ void __launch_bounds__(256)
rbwd_wsplit_kernel(const float* __restrict__ w_r, int N, int NP16, int d, __nv_bfloat16* __restrict__ bdx) {
    pdl_wait();
    pdl_launch();
    const int64_t n_el = (int64_t)NP16 * d;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < n_el; q += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(q / d);
        const int c = (int)(q - (int64_t)e * d);
        __nv_bfloat16 w[3];
        split3(e < N ? w_r[(int64_t)e * d + c] : 0.f, w[0], w[1], w[2]);
        const int part[6] = {0, 1, 0, 2, 1, 0};   // the W_r part each K segment multiplies
#pragma unroll
        for (int sg = 0; sg < 6; ++sg) bdx[((int64_t)sg * NP16 + e) * d + c] = w[part[sg]];
    }
}

// part_db[chunk][e] = sum over the chunk's tokens of dh[t][e] (fp32, in order)
__global__ void __launch_bounds__(128)
rbwd_db_kernel(const float* __restrict__ dh, int64_t T, int N, int64_t chunk, float* __restrict__ part_db) {
    pdl_wait();
    pdl_launch();
    const int e = threadIdx.x;
    if (e >= N) return;
    const int64_t t0 = (int64_t)blockIdx.x * chunk, t1 = min(T, t0 + chunk);
    float acc = 0.f;
    constexpr int B = 64;   // loads in flight, then added in token order
    int64_t t = t0;
    for (; t + B <= t1; t += B) {
        float v[B];
#pragma unroll
        for (int j = 0; j < B; ++j) v[j] = dh[(t + j) * N + e];
#pragma unroll
        for (int j = 0; j < B; ++j) acc += v[j];
    }
    for (; t < t1; ++t) acc += dh[t * N + e];
    part_db[(int64_t)blockIdx.x * N + e] = acc;
}

// dw[e][c] = sum over chunks (in order) of the three parts' partial products,
// db[e] = sum over chunks of part_db; fp64
__global__ void __launch_bounds__(256)
rbwd_reduce_tc_kernel(const float* __restrict__ part, const float* __restrict__ part_db, int nchunk, int N, int NP16,
                      int d, float* __restrict__ dw, float* __restrict__ db) {
    pdl_wait();
    pdl_launch();
    const int64_t n = (int64_t)N * d;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < n + N; q += (int64_t)gridDim.x * blockDim.x) {
        if (q < n) {
            if (!dw) continue;
            const int e = (int)(q / d);
            const int c = (int)(q - (int64_t)e * d);
            double acc = 0.0;
            for (int ch = 0; ch < nchunk; ++ch) {
                const float* pc = part + (int64_t)ch * 3 * NP16 * d;
#pragma unroll
                for (int j = 0; j < 3; ++j) acc += (double)pc[((int64_t)j * NP16 + e) * d + c];
            }
            dw[q] = (float)acc;
        } else if (db) {
            const int e = (int)(q - n);
            double acc = 0.0;
            for (int ch = 0; ch < nchunk; ++ch) acc += (double)part_db[(int64_t)ch * N + e];
            db[e] = (float)acc;
        }
    }
}

}  // namespace

int router_bwd_chunks(int64_t T) { return (int)((T + kBwdChunk - 1) / kBwdChunk); }
int router_bwd_np16(int N) { return (N + 15) / 16 * 16; }
int64_t router_bwd_tc_chunk(int64_t T) {
    int64_t c = (T + 127) / 128;   // at most 128 chunks (the weight GEMM's group limit)
    c = (c + 63) / 64 * 64;
    return c < kBwdChunk ? kBwdChunk : c;
}
int router_bwd_tc_chunks(int64_t T) {
    const int64_t c = router_bwd_tc_chunk(T);
    return (int)((T + c - 1) / c);
}

cudaError_t launch_router_backward(const RouterBwdArgs& a, cudaStream_t s) {
    if (a.T <= 0) {   // no tokens: every gradient is zero
        cudaError_t e = cudaSuccess;
        if (a.dw) e = cudaMemsetAsync(a.dw, 0, sizeof(float) * a.N * a.d, s);
        if (e == cudaSuccess && a.db) e = cudaMemsetAsync(a.db, 0, sizeof(float) * a.N, s);
        return e;
    }
    cudaError_t err = launch_k(router_bwd_dh_kernel, dim3((unsigned)((a.T + 8 * kDhTokens - 1) / (8 * kDhTokens))),
                               dim3(256), 0, s, 1, a.probs,
                               a.idx, a.gate, a.dgate, a.f, a.alpha, a.T, a.N, a.k, a.dh);
    if (err != cudaSuccess) return err;
    if (a.dtype == MOE_BF16 && a.tc_adx && (a.dw || a.db || a.dx)) {
        // the contractions on the tensor cores
        const int NP16 = router_bwd_np16(a.N);
        const int64_t chunk = router_bwd_tc_chunk(a.T);
        const int nchunk = router_bwd_tc_chunks(a.T);
        const int64_t n_el = a.T * (NP16 / 8);   // a thread per eight experts of a token
        const unsigned sg = (unsigned)((n_el + 255) / 256 < 8192 ? (n_el + 255) / 256 : 8192);
        if ((err = launch_k(rbwd_split_kernel, dim3(sg), dim3(256), 0, s, 1, static_cast<const float*>(a.dh), a.T,
                            a.N, NP16, reinterpret_cast<__nv_bfloat16*>(a.tc_adx),
                            reinterpret_cast<__nv_bfloat16*>(a.tc_adw), a.tc_offs, chunk, nchunk)) != cudaSuccess)
            return err;
        if (a.dx) {
            const int64_t w_el = (int64_t)NP16 * a.d;
            const unsigned wg = (unsigned)((w_el + 255) / 256 < 4096 ? (w_el + 255) / 256 : 4096);
            if ((err = launch_k(rbwd_wsplit_kernel, dim3(wg), dim3(256), 0, s, 1, a.w_r, a.N, NP16, a.d,
                                reinterpret_cast<__nv_bfloat16*>(a.tc_bdx))) != cudaSuccess)
                return err;
            if ((err = launch_tc_rows_f32(a.tc_adx, a.T, 6 * NP16, a.tc_bdx, a.d, a.tc_offs, a.dx, a.status, s)) !=
                cudaSuccess)
                return err;
        }
        if (a.dw || a.db) {
            if (a.dw && (err = launch_tc_weights_f32(a.tc_adw, a.T, 3 * NP16, a.x, a.d, a.tc_offs + 2, nchunk,
                                                     a.tc_part, a.status, s)) != cudaSuccess)
                return err;
            if ((err = launch_k(rbwd_db_kernel, dim3((unsigned)nchunk), dim3(128), 0, s, 1,
                                static_cast<const float*>(a.dh), a.T, a.N, chunk, a.part_db)) != cudaSuccess)
                return err;
            const int64_t n = (int64_t)a.N * a.d + a.N;
            const unsigned rg = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
            if ((err = launch_k(rbwd_reduce_tc_kernel, dim3(rg), dim3(256), 0, s, 1,
                                static_cast<const float*>(a.tc_part), static_cast<const float*>(a.part_db), nchunk,
                                a.N, NP16, a.d, a.dw, a.db)) != cudaSuccess)
                return err;
        }
        return cudaSuccess;
    }
    if (a.dw || a.db) {
        const int nchunk = router_bwd_chunks(a.T);
        const dim3 g((unsigned)nchunk, (unsigned)((a.N + 31) / 32), (unsigned)((a.d + 127) / 128));
        err = a.dtype == MOE_BF16
                  ? launch_k(router_bwd_dw_kernel<__nv_bfloat16>, g, dim3(256), 0, s, 1,
                             static_cast<const float*>(a.dh), reinterpret_cast<const __nv_bfloat16*>(a.x), a.T, a.N,
                             a.d, a.part_dw, a.part_db)
                  : launch_k(router_bwd_dw_kernel<float>, g, dim3(256), 0, s, 1, static_cast<const float*>(a.dh),
                             reinterpret_cast<const float*>(a.x), a.T, a.N, a.d, a.part_dw, a.part_db);
        if (err != cudaSuccess) return err;
        const int64_t n = (int64_t)a.N * a.d + a.N;
        const unsigned rg = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
        err = launch_k(router_bwd_reduce_kernel, dim3(rg), dim3(256), 0, s, 1, static_cast<const float*>(a.part_dw),
                       static_cast<const float*>(a.part_db), nchunk, a.N, a.d, a.dw, a.db);
        if (err != cudaSuccess) return err;
    }
    if (a.dx) {
        const dim3 g((unsigned)((a.T + 63) / 64), (unsigned)((a.d + 127) / 128));
        err = launch_k(router_bwd_dx_kernel, g, dim3(256), 0, s, 1, static_cast<const float*>(a.dh), a.w_r, a.T, a.N,
                       a.d, a.dx);
    }
    return err;
}

}  // namespace moe
