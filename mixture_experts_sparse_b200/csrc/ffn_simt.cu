// Expert FFN on the FP32 pipe, for fp32 layers (the tensor cores' bf16/tf32
// inputs cannot hold an fp32 layer to its tolerance), plus the dispatcher that
// sends bf16 layers to the tcgen05 grouped GEMM.
//
// Same mathematics as the tensor-core path: per expert e and compact row r of e,
// H = act(A W1[e]^T + b1[e]) (or the SwiGLU product), then Y = H W2[e]^T + b2[e]
// ("From Switch Transformer to GLaM", FFN(x) = W2 s(W1 x); CMU 10-423 Lecture
// 16, section 2.3, SwiGLU expert).  A 64x64 output tile per block, 4x4 per
// thread, K staged through shared memory in chunks of 32.  Grid = (m-tiles up to
// the capacity C, n-tiles, experts); blocks past an expert's kept rows return.
#include "common.cuh"

namespace moe {


namespace {

constexpr int TS = 64;
constexpr int KC = 32;

enum { SIMT_RELU = 0, SIMT_SWIGLU = 1, SIMT_BIAS = 2 };

template <int MODE>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets, int K, int n_dim,
                 const float* __restrict__ B, const float* __restrict__ B3, const float* __restrict__ bias,
                 const float* __restrict__ bias3, float* __restrict__ out) {
    pdl_wait();
    pdl_launch();
    const int e = blockIdx.z;
    const int row0 = offsets[e];
    const int rows = offsets[e + 1] - row0;
    const int m0 = blockIdx.x * TS;
    if (m0 >= rows) return;
    const int n0 = blockIdx.y * TS;
    const float* Be = B + (int64_t)e * n_dim * K;
    const float* B3e = (MODE == SIMT_SWIGLU) ? B3 + (int64_t)e * n_dim * K : nullptr;

    __shared__ float As[KC][TS + 4];
    __shared__ float Bs[KC][TS + 4];
    __shared__ float B3s[(MODE == SIMT_SWIGLU) ? KC : 1][TS + 4];

    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    float acc[4][4] = {};
    float acc3[4][4] = {};
    // the next K chunk is loaded into registers while the current one is used
    constexpr int PER = TS * KC / 256;
    float pa[PER], pb[PER], pb3[PER];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int l = 0; l < PER; ++l) {
            const int q = tid + 256 * l;
            const int rr = q / KC, kk = q % KC;
            const int m = m0 + rr, kx = k0 + kk, n = n0 + rr;
            pa[l] = (m < rows && kx < K) ? A[(int64_t)(row0 + m) * K + kx] : 0.f;
            pb[l] = (n < n_dim && kx < K) ? Be[(int64_t)n * K + kx] : 0.f;
            if (MODE == SIMT_SWIGLU) pb3[l] = (n < n_dim && kx < K) ? B3e[(int64_t)n * K + kx] : 0.f;
        }
    };
    fetch(0);
    for (int k0 = 0; k0 < K; k0 += KC) {
#pragma unroll
        for (int l = 0; l < PER; ++l) {
            const int q = tid + 256 * l;
            const int rr = q / KC, kk = q % KC;
            As[kk][rr] = pa[l];
            Bs[kk][rr] = pb[l];
            if (MODE == SIMT_SWIGLU) B3s[kk][rr] = pb3[l];
        }
        __syncthreads();
        if (k0 + KC < K) fetch(k0 + KC);
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) {
            float a[4], b[4], b3[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                b[i] = Bs[kk][tx * 4 + i];
                if (MODE == SIMT_SWIGLU) b3[i] = B3s[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
                    if (MODE == SIMT_SWIGLU) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int m = m0 + ty * 4 + i;
        if (m >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int n = n0 + tx * 4 + j;
            if (n >= n_dim) continue;
            float v = acc[i][j] + (bias ? bias[(int64_t)e * n_dim + n] : 0.f);
            if (MODE == SIMT_RELU) {
                v = fmaxf(v, 0.f);
            } else if (MODE == SIMT_SWIGLU) {
                float g = acc3[i][j] + (bias3 ? bias3[(int64_t)e * n_dim + n] : 0.f);
                v = (v / (1.f + expf(-v))) * g;
            }
            out[(int64_t)(row0 + m) * n_dim + n] = v;
        }
    }
}

cudaError_t launch_expert_ffn_simt(const FfnArgs& a, cudaStream_t s) {
    if (a.C <= 0) return cudaSuccess;
    const unsigned mt = (unsigned)((a.C + TS - 1) / TS);
    const float* xe = reinterpret_cast<const float*>(a.xe);
    float* h = reinterpret_cast<float*>(a.h);
    dim3 g1(mt, (unsigned)((a.d_ff + TS - 1) / TS), (unsigned)a.N);
    const float* none = nullptr;
    cudaError_t err =
        a.act == MOE_SWIGLU
            ? launch_k(simt_gemm_kernel<SIMT_SWIGLU>, g1, dim3(256), 0, s, 1, xe, a.offsets, a.d, a.d_ff,
                       reinterpret_cast<const float*>(a.w1), reinterpret_cast<const float*>(a.w3),
                       reinterpret_cast<const float*>(a.b1), reinterpret_cast<const float*>(a.b3), h)
            : launch_k(simt_gemm_kernel<SIMT_RELU>, g1, dim3(256), 0, s, 1, xe, a.offsets, a.d, a.d_ff,
                       reinterpret_cast<const float*>(a.w1), none, reinterpret_cast<const float*>(a.b1), none, h);
    if (err != cudaSuccess) return err;
    if (a.mid_event && (err = cudaEventRecord((cudaEvent_t)a.mid_event, s)) != cudaSuccess) return err;
    dim3 g2(mt, (unsigned)((a.d + TS - 1) / TS), (unsigned)a.N);
    return launch_k(simt_gemm_kernel<SIMT_BIAS>, g2, dim3(256), 0, s, 1, static_cast<const float*>(h), a.offsets,
                    a.d_ff, a.d, reinterpret_cast<const float*>(a.w2), none, reinterpret_cast<const float*>(a.b2), none,
                    reinterpret_cast<float*>(a.ye));
}

}  // namespace

cudaError_t launch_expert_ffn(const FfnArgs& a, cudaStream_t s) {
    if (a.dtype == MOE_BF16) return launch_expert_ffn_tc(a, s);
    return launch_expert_ffn_simt(a, s);
}

}  // namespace moe
