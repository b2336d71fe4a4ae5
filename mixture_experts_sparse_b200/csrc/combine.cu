// Gate-scaled combine back to token order:
//   out_t = sum over kept r of gate[t, r] * ye[offsets[idx[t, r]] + pos[t, r]]
// accumulated in fp32 in rank order and rounded once; a token whose every
// assignment was dropped outputs zero (its residual connection, outside the
// layer, carries it).  "From Switch Transformer to GLaM": y = p_{i*} E_{i*}(x)
// for top-1 and y = w1 E_{i1}(x) + w2 E_{i2}(x) for top-2, "Expert Capacity and
// Token Dropping" (an overflowing token skips the expert FFN).
// One warp per token, 16-byte vector loads/stores: an HBM-bound gather.
//
// For one shard of a routing group pos holds group-wide claim numbers; the
// shard's rows of expert e hold its kept rank-0 claims (numbers base0[e] ...)
// and then its kept rank-1 claims (numbers base1[e] ...), so the row of a kept
// claim p is p - base0[e] (rank 0) or kept0[e] + p - base1[e] (rank 1), kept0
// being how many of the shard's rank-0 claims on e fall below C.
#include "common.cuh"

namespace moe {
namespace {

template <typename XT>
__global__ void __launch_bounds__(256)
combine_kernel(const XT* __restrict__ ye, const int32_t* __restrict__ idx, const int32_t* __restrict__ pos,
               const uint8_t* __restrict__ drop, const float* __restrict__ gate,
               const int32_t* __restrict__ offsets, const int32_t* __restrict__ claim_base,
               const int32_t* __restrict__ counts, int C, int N, int64_t T, int d, int k, XT* __restrict__ out) {
    constexpr int VEC = 16 / sizeof(XT);
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    int64_t row[2] = {-1, -1};
    float g[2] = {0.f, 0.f};
    for (int r = 0; r < k; ++r) {
        const int64_t a = t * k + r;
        if (!drop[a]) {
            const int e = idx[a];
            int local = pos[a];
            if (claim_base)
                local = r == 0 ? local - claim_base[e]
                               : kept_after(claim_base[e], counts[e], C) + local - claim_base[N + e];
            row[r] = (int64_t)offsets[e] + local;
            g[r] = gate[a];
        }
    }
    XT* dst = out + t * (int64_t)d;
    if (((size_t)d * sizeof(XT)) % 16 == 0) {
        for (int c = lane * VEC; c < d; c += 32 * VEC) {
            float acc[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
            for (int r = 0; r < k; ++r) {
                if (row[r] < 0) continue;
                uint4 v = __ldg(reinterpret_cast<const uint4*>(ye + row[r] * d + c));
                const XT* xv = reinterpret_cast<const XT*>(&v);
#pragma unroll
                for (int j = 0; j < VEC; ++j) acc[j] = fmaf(g[r], Elem<XT>::to_f(xv[j]), acc[j]);
            }
            XT o[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) o[j] = Elem<XT>::from_f(acc[j]);
            *reinterpret_cast<uint4*>(dst + c) = *reinterpret_cast<uint4*>(o);
        }
    } else {
        for (int c = lane; c < d; c += 32) {
            float acc = 0.f;
            for (int r = 0; r < k; ++r)
                if (row[r] >= 0) acc = fmaf(g[r], Elem<XT>::to_f(ye[row[r] * d + c]), acc);
            dst[c] = Elem<XT>::from_f(acc);
        }
    }
}

// dL/dgate[t, r] = <dout_t, ye[offsets[idx[t,r]] + pos[t,r]]> for a kept
// assignment, 0 for a dropped one: the gate's gradient for the router backward
// (out_t = sum_r gate_{t,r} E(x_t), "From Switch Transformer to GLaM").  One
// warp per assignment, fp32 accumulation, a fixed shuffle tree.
template <typename XT>
__global__ void __launch_bounds__(256)
gate_grad_kernel(const XT* __restrict__ dout, const XT* __restrict__ ye, const int32_t* __restrict__ idx,
                 const int32_t* __restrict__ pos, const uint8_t* __restrict__ drop,
                 const int32_t* __restrict__ offsets, int64_t T, int d, int k, float* __restrict__ dgate) {
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t a = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (a >= T * k) return;
    const int64_t t = a / k;
    float acc = 0.f;
    if (!drop[a]) {
        const int64_t row = (int64_t)offsets[idx[a]] + pos[a];
        const XT* g = dout + t * (int64_t)d;
        const XT* y = ye + row * (int64_t)d;
        for (int c = lane; c < d; c += 32) acc = fmaf(Elem<XT>::to_f(g[c]), Elem<XT>::to_f(y[c]), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dgate[a] = acc;
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((a.T + 7) / 8);
    if (a.dtype == MOE_BF16)
        return launch_k(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.ye), a.idx, a.pos, a.drop, a.gate, a.offsets,
                        a.claim_base, a.counts, a.C, a.N, a.T, a.d, a.k, reinterpret_cast<__nv_bfloat16*>(a.out));
    return launch_k(combine_kernel<float>, dim3(grid), dim3(256), 0, s, 1, reinterpret_cast<const float*>(a.ye), a.idx,
                    a.pos, a.drop, a.gate, a.offsets, a.claim_base, a.counts, a.C, a.N, a.T, a.d, a.k,
                    reinterpret_cast<float*>(a.out));
}

cudaError_t launch_gate_grad(const GateGradArgs& a, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((a.T * a.k + 7) / 8);
    if (a.dtype == MOE_BF16)
        return launch_k(gate_grad_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.dout), reinterpret_cast<const __nv_bfloat16*>(a.ye),
                        a.idx, a.pos, a.drop, a.offsets, a.T, a.d, a.k, a.dgate);
    return launch_k(gate_grad_kernel<float>, dim3(grid), dim3(256), 0, s, 1, reinterpret_cast<const float*>(a.dout),
                    reinterpret_cast<const float*>(a.ye), a.idx, a.pos, a.drop, a.offsets, a.T, a.d, a.k, a.dgate);
}

}  // namespace moe
