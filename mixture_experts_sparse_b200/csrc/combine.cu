// Gate-scaled combine back to token order:
//   out_t = sum over kept r of gate[t, r] * ye[offsets[idx[t, r]] + pos[t, r]]
// accumulated in fp32 in rank order and rounded once; a token whose every
// assignment was dropped outputs zero (its residual connection, outside the
// layer, carries it).  "From Switch Transformer to GLaM": y = p_{i*} E_{i*}(x)
// for top-1 and y = w1 E_{i1}(x) + w2 E_{i2}(x) for top-2, "Expert Capacity and
// Token Dropping" (an overflowing token skips the expert FFN).
// 16-byte vector loads/stores: an HBM-bound gather.
//
// For one shard of a routing group pos holds group-wide claim numbers; the
// shard's rows of expert e hold its kept rank-0 claims (numbers base0[e] ...)
// and then its kept rank-1 claims (numbers base1[e] ...), so the row of a kept
// claim p is p - base0[e] (rank 0) or kept0[e] + p - base1[e] (rank 1), kept0
// being how many of the shard's rank-0 claims on e fall below C.
#include "common.cuh"

namespace moe {
namespace {

// One warp per kCombineTokens consecutive tokens: lanes 0 .. kCombineTokens*k-1
// each locate one assignment's row and gate (one dependent chain of loads per
// warp instead of one per token), then the warp combines the tokens one after
// another with all of a token's 16-byte row loads (up to kCombineUnroll
// chunks per lane per row) in flight before its first store.  With a warp per
// token, 4096 blocks of 256 threads each lived about a microsecond at top-2
// sizes and block launches bounded the kernel.
constexpr int kCombineTokens = 4;
constexpr int kCombineUnroll = 4;

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
    const int64_t t0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * kCombineTokens;
    if (t0 >= T) return;
    int64_t my_row = -1;   // lane i < kCombineTokens * k: token t0 + i / k, rank i % k (-1: dropped)
    float my_g = 0.f;
    if (lane < kCombineTokens * k) {
        const int64_t t = t0 + lane / k;
        const int r = lane - (lane / k) * k;
        const int64_t a = t * k + r;
        if (t < T && !drop[a]) {
            const int e = idx[a];
            int local = pos[a];
            if (claim_base)
                local = r == 0 ? local - claim_base[e]
                               : kept_after(claim_base[e], counts[e], C) + local - claim_base[N + e];
            my_row = (int64_t)offsets[e] + local;
            my_g = gate[a];
        }
    }
#pragma unroll 1
    for (int i = 0; i < kCombineTokens; ++i) {
        const int64_t t = t0 + i;
        if (t >= T) break;   // warp-uniform
        int64_t row[2];
        float g[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int src = i * k + (r < k ? r : 0);
            row[r] = __shfl_sync(0xffffffffu, my_row, src);
            g[r] = __shfl_sync(0xffffffffu, my_g, src);
            if (r >= k) row[r] = -1;
        }
        XT* dst = out + t * (int64_t)d;
        if (((size_t)d * sizeof(XT)) % 16 == 0) {
            for (int c0 = lane * VEC; c0 < d; c0 += 32 * VEC * kCombineUnroll) {
                uint4 v[2][kCombineUnroll];
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int u = 0; u < kCombineUnroll; ++u) {
                        const int c = c0 + u * 32 * VEC;
                        v[r][u] = (row[r] >= 0 && c < d)
                                      ? __ldg(reinterpret_cast<const uint4*>(ye + row[r] * d + c))
                                      : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    const int c = c0 + u * 32 * VEC;
                    if (c >= d) break;
                    float acc[VEC];
#pragma unroll
                    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {   // rank order, one rounding at the end
                        if (row[r] < 0) continue;
                        const XT* xv = reinterpret_cast<const XT*>(&v[r][u]);
#pragma unroll
                        for (int j = 0; j < VEC; ++j) acc[j] = fmaf(g[r], Elem<XT>::to_f(xv[j]), acc[j]);
                    }
                    XT o[VEC];
#pragma unroll
                    for (int j = 0; j < VEC; ++j) o[j] = Elem<XT>::from_f(acc[j]);
                    *reinterpret_cast<uint4*>(dst + c) = *reinterpret_cast<uint4*>(o);
                }
            }
        } else {
            for (int c = lane; c < d; c += 32) {
                float acc = 0.f;
                for (int r = 0; r < 2; ++r)
                    if (row[r] >= 0) acc = fmaf(g[r], Elem<XT>::to_f(ye[row[r] * d + c]), acc);
                dst[c] = Elem<XT>::from_f(acc);
            }
        }
    }
}

// dL/dgate[t, r] = <dout_t, ye[offsets[idx[t,r]] + pos[t,r]]> for a kept
// assignment, 0 for a dropped one: the gate's gradient for the router backward
// (out_t = sum_r gate_{t,r} E(x_t), "From Switch Transformer to GLaM").  A warp
// per kGradAssign assignments, laid out like the combine: lanes locate the
// rows together, then per assignment every 16-byte load of both rows is in
// flight before the fp32 products are summed; a fixed shuffle tree finishes
// each dot product.
constexpr int kGradAssign = 4;

template <typename XT>
__global__ void __launch_bounds__(256)
gate_grad_kernel(const XT* __restrict__ dout, const XT* __restrict__ ye, const int32_t* __restrict__ idx,
                 const int32_t* __restrict__ pos, const uint8_t* __restrict__ drop,
                 const int32_t* __restrict__ offsets, int64_t T, int d, int k, float* __restrict__ dgate) {
    constexpr int VEC = 16 / sizeof(XT);
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t n_assign = T * k;
    const int64_t a0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * kGradAssign;
    if (a0 >= n_assign) return;
    int64_t my_row = -1;   // lane i < kGradAssign: assignment a0 + i's row of ye (-1: dropped)
    if (lane < kGradAssign && a0 + lane < n_assign && !drop[a0 + lane])
        my_row = (int64_t)offsets[idx[a0 + lane]] + pos[a0 + lane];
#pragma unroll 1
    for (int i = 0; i < kGradAssign; ++i) {
        const int64_t a = a0 + i;
        if (a >= n_assign) break;   // warp-uniform
        const int64_t row = __shfl_sync(0xffffffffu, my_row, i);
        float acc = 0.f;
        if (row >= 0) {
            const XT* g = dout + (a / k) * (int64_t)d;
            const XT* y = ye + row * (int64_t)d;
            if (((size_t)d * sizeof(XT)) % 16 == 0) {
                for (int c0 = lane * VEC; c0 < d; c0 += 32 * VEC * kCombineUnroll) {
                    uint4 vg[kCombineUnroll], vy[kCombineUnroll];
#pragma unroll
                    for (int u = 0; u < kCombineUnroll; ++u) {
                        const int c = c0 + u * 32 * VEC;
                        vg[u] = c < d ? __ldg(reinterpret_cast<const uint4*>(g + c)) : make_uint4(0, 0, 0, 0);
                        vy[u] = c < d ? __ldg(reinterpret_cast<const uint4*>(y + c)) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < kCombineUnroll; ++u) {
                        const XT* xg = reinterpret_cast<const XT*>(&vg[u]);
                        const XT* xy = reinterpret_cast<const XT*>(&vy[u]);
#pragma unroll
                        for (int j = 0; j < VEC; ++j) acc = fmaf(Elem<XT>::to_f(xg[j]), Elem<XT>::to_f(xy[j]), acc);
                    }
                }
            } else {
                for (int c = lane; c < d; c += 32) acc = fmaf(Elem<XT>::to_f(g[c]), Elem<XT>::to_f(y[c]), acc);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) dgate[a] = acc;
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((a.T + 8 * kCombineTokens - 1) / (8 * kCombineTokens));
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
    const unsigned grid = (unsigned)((a.T * a.k + 8 * kGradAssign - 1) / (8 * kGradAssign));
    if (a.dtype == MOE_BF16)
        return launch_k(gate_grad_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.dout), reinterpret_cast<const __nv_bfloat16*>(a.ye),
                        a.idx, a.pos, a.drop, a.offsets, a.T, a.d, a.k, a.dgate);
    return launch_k(gate_grad_kernel<float>, dim3(grid), dim3(256), 0, s, 1, reinterpret_cast<const float*>(a.dout),
                    reinterpret_cast<const float*>(a.ye), a.idx, a.pos, a.drop, a.offsets, a.T, a.d, a.k, a.dgate);
}

}  // namespace moe
