// Expert parallelism: the experts of one layer spread over G GPUs (E = N / G
// experts per GPU, expert e on GPU e / E), with the dispatch all-to-all and the
// combine all-to-all of "From Switch Transformer to GLaM" (section All-to-All:
// the dispatch moves each token from its data-parallel home to the device of
// its expert, the combine moves the expert output back) and CMU 10-423
// Lecture 16, section 6.2 (the all-to-all volume per GPU per layer).
//
// Every GPU keeps its own tokens, routing and capacity (a routing group per
// GPU, as in the pages' data-parallel x expert-parallel layout).  After the
// local route and slot claim, the compact rows of expert e are
// [offsets[e], offsets[e + 1]) of the source GPU.  One small all-gather of every
// GPU's kept[N] fixes where everything lands:
//   receiver h, local expert j (e = h E + j): rows of source 0, then of source
//   1, ... ; recv_offsets[j] = sum over j' < j, all sources s of kept_s[h E + j']
//   source g writes its rows of e starting at
//   dst_start[e] = recv_offsets_h[j] + sum over s < g of kept_s[e].
// The dispatch kernel reads each kept row's token straight from x (the gather
// fused into the transfer) and stores it, with the row's return address
// (source GPU, destination row, gate), into the owner's receive buffers
// through peer pointers: plain loads from local memory, plain stores to peer
// memory.  The receiver's grouped GEMM epilogue then sends every result row
// back the same way (gemm_tc.cu, scatter epilogue with per-row destination
// GPU); ep_return_kernel does it for layers whose expert FFN has no fused
// epilogue (fp32).
#include "common.cuh"

namespace moe {
namespace {

// dst_start [N] (this GPU as a source) and recv_offsets [E + 1] (this GPU as a
// receiver) from kept_all [G][N].  One block; N <= 128.
__global__ void ep_layout_kernel(int G, int rank, int N, const int32_t* __restrict__ kept_all,
                                 int32_t* __restrict__ dst_start, int32_t* __restrict__ recv_offsets) {
    pdl_wait();
    pdl_launch();
    const int E = N / G;
    __shared__ int32_t tot[128];    // rows every source sends to expert e
    __shared__ int32_t start[128];  // first receive row of expert e on its owner
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        int32_t t = 0;
        for (int s = 0; s < G; ++s) t += kept_all[(int64_t)s * N + e];
        tot[e] = t;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        const int h = e / E;
        int32_t st = 0;
        for (int e2 = h * E; e2 < e; ++e2) st += tot[e2];
        start[e] = st;
        int32_t before = 0;
        for (int s = 0; s < rank; ++s) before += kept_all[(int64_t)s * N + e];
        dst_start[e] = st + before;
    }
    __syncthreads();
    for (int j = threadIdx.x; j <= E; j += blockDim.x) {
        const int e = rank * E + j;
        recv_offsets[j] = j < E ? start[e] : (E > 0 ? start[e - 1] + tot[e - 1] : 0);
    }
}

// expert of compact row r: the e with offsets[e] <= r < offsets[e + 1]
__device__ __forceinline__ int row_expert(const int32_t* off, int N, int r) {
    int lo = 0, hi = N;   // off[lo] <= r < off[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= r) lo = mid;
        else hi = mid;
    }
    return lo;
}

struct EpPeers {
    void* const* recv_x;          // [G] receive rows [R_recv, d] on each GPU
    int32_t* const* recv_rank;    // [G] source GPU of each received row
    int32_t* const* recv_row;     // [G] where its result goes on the source (token, or compact row)
    float* const* recv_gate;      // [G] its gate
};

// One warp per compact row of this GPU (rows beyond offsets[N] exit), then,
// for top-1, one warp per token zeroes the output rows of dropped tokens.
template <typename XT>
__global__ void __launch_bounds__(256)
ep_dispatch_kernel(const XT* __restrict__ x, int64_t T, int d, int N, int G, int rank, int k,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ row_token,
                   const float* __restrict__ row_gate, const int32_t* __restrict__ dst_start, EpPeers peers,
                   int64_t row_blocks, const uint8_t* __restrict__ drop, XT* __restrict__ out) {
    pdl_wait();
    pdl_launch();
    __shared__ int32_t s_off[129];
    for (int i = threadIdx.x; i <= N; i += blockDim.x) s_off[i] = offsets[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const size_t bytes = (size_t)d * sizeof(XT);
    if ((int64_t)blockIdx.x < row_blocks) {
        const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
        if (r >= s_off[N]) return;
        const int e = row_expert(s_off, N, (int)r);
        const int E = N / G;
        const int h = e / E;
        const int64_t drow = (int64_t)dst_start[e] + (r - s_off[e]);
        const int64_t t = row_token[r];
        if (lane == 0) {
            peers.recv_rank[h][drow] = rank;
            peers.recv_row[h][drow] = (int32_t)(k == 1 ? t : r);   // top-1: the token's out row; top-2: its ye row
            peers.recv_gate[h][drow] = row_gate[r];
        }
        const char* src = reinterpret_cast<const char*>(x + t * (int64_t)d);
        char* dst = reinterpret_cast<char*>(peers.recv_x[h]) + drow * (int64_t)bytes;
        if (bytes % 16 == 0) {
            for (size_t o = (size_t)lane * 16; o < bytes; o += 32 * 16)
                *reinterpret_cast<uint4*>(dst + o) = __ldg(reinterpret_cast<const uint4*>(src + o));
        } else {
            for (size_t o = (size_t)lane * sizeof(XT); o < bytes; o += 32 * sizeof(XT))
                *reinterpret_cast<XT*>(dst + o) = *reinterpret_cast<const XT*>(src + o);
        }
        __threadfence_system();   // the stores reach the peer before this kernel is seen to finish
        return;
    }
    // top-1: a dropped token's output row is zero (its results arrive from the
    // experts' GPUs only for kept tokens)
    if (out == nullptr) return;
    const int64_t t = ((int64_t)blockIdx.x - row_blocks) * 8 + (threadIdx.x >> 5);
    if (t >= T || !drop[t]) return;
    char* dst = reinterpret_cast<char*>(out + t * (int64_t)d);
    if (bytes % 16 == 0) {
        for (size_t o = (size_t)lane * 16; o < bytes; o += 32 * 16)
            *reinterpret_cast<uint4*>(dst + o) = make_uint4(0, 0, 0, 0);
    } else {
        for (int j = lane; j < d; j += 32) out[t * (int64_t)d + j] = XT(0.f);
    }
}

// Result rows back to their source GPUs: out_ptrs[recv_rank[r]] row recv_row[r]
// = gate (top-1) or 1 (top-2) times ye[r].  One warp per received row.
template <typename XT>
__global__ void __launch_bounds__(256)
ep_return_kernel(const XT* __restrict__ ye, const int32_t* __restrict__ recv_offsets, int E, int d,
                 const int32_t* __restrict__ recv_rank, const int32_t* __restrict__ recv_row,
                 const float* __restrict__ recv_gate, void* const* __restrict__ out_ptrs) {
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= recv_offsets[E]) return;
    const float g = recv_gate ? recv_gate[r] : 1.f;
    XT* dst = reinterpret_cast<XT*>(out_ptrs[recv_rank[r]]) + (int64_t)recv_row[r] * d;
    const XT* src = ye + r * (int64_t)d;
    for (int c = lane; c < d; c += 32) dst[c] = Elem<XT>::from_f(g * Elem<XT>::to_f(src[c]));
    __threadfence_system();
}

}  // namespace

cudaError_t launch_ep_layout(int G, int rank, int N, const int32_t* kept_all, int32_t* dst_start,
                             int32_t* recv_offsets, cudaStream_t s) {
    return launch_k(ep_layout_kernel, dim3(1), dim3(128), 0, s, 1, G, rank, N, kept_all, dst_start, recv_offsets);
}

cudaError_t launch_ep_dispatch(const EpDispatchArgs& a, cudaStream_t s) {
    const int64_t row_blocks = (a.R_cap + 7) / 8;
    const int64_t tok_blocks = (a.k == 1 && a.out) ? (a.T + 7) / 8 : 0;
    if (row_blocks + tok_blocks == 0) return cudaSuccess;
    EpPeers peers{a.recv_x, a.recv_rank, a.recv_row, a.recv_gate};
    const dim3 grid((unsigned)(row_blocks + tok_blocks));
    if (a.dtype == MOE_BF16)
        return launch_k(ep_dispatch_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.x), a.T, a.d, a.N, a.G, a.rank, a.k, a.offsets,
                        a.row_token, a.row_gate, a.dst_start, peers, row_blocks, a.drop,
                        reinterpret_cast<__nv_bfloat16*>(a.out));
    return launch_k(ep_dispatch_kernel<float>, grid, dim3(256), 0, s, 1, reinterpret_cast<const float*>(a.x), a.T, a.d,
                    a.N, a.G, a.rank, a.k, a.offsets, a.row_token, a.row_gate, a.dst_start, peers, row_blocks, a.drop,
                    reinterpret_cast<float*>(a.out));
}

cudaError_t launch_ep_return(int dtype, const void* ye, const int32_t* recv_offsets, int E, int d, int64_t R_cap,
                             const int32_t* recv_rank, const int32_t* recv_row, const float* recv_gate,
                             void* const* out_ptrs, cudaStream_t s) {
    if (R_cap <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((R_cap + 7) / 8));
    if (dtype == MOE_BF16)
        return launch_k(ep_return_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(ye), recv_offsets, E, d, recv_rank, recv_row,
                        recv_gate, out_ptrs);
    return launch_k(ep_return_kernel<float>, grid, dim3(256), 0, s, 1, reinterpret_cast<const float*>(ye),
                    recv_offsets, E, d, recv_rank, recv_row, recv_gate, out_ptrs);
}

}  // namespace moe
