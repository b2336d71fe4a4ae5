// Shared device/host helpers of libmoe_b200 (internal header).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Tokens per block of the dispatch scan (dispatch.cu); the look-back state
// holds one word per (scan block, rank, expert).
constexpr int kScanTokens = 1024;

// Argument checks every entry point that takes a moe_config runs first
// (MOE_OK or the status to return); defined in api.cu.
int32_t validate_config(const moe_config* c);

// ---- workspace header (first 256 bytes of every workspace) ----------------
struct WsHeader {
    int32_t status;        // latched moe_status of device-side failures
    int32_t scan_ticket;   // dynamic block index of the dispatch scan
    int32_t scan_done;     // finished-block counter of the dispatch scan
    int32_t route_ticket;  // finished-CTA counter of the tensor-core router
    int32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

// Default limit of every device-side bounded wait: far above any legitimate
// wait (microseconds), low enough that a wedged wait returns promptly.
constexpr long long kWaitLimitNs = 2000000000LL;

__device__ __forceinline__ long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return (long long)t;
}

// 2^x in one MUFU instruction (PTX ex2.approx.ftz.f32: relative error about
// 2^-22; results below 2^-126 flush to zero, 2^-inf = 0).  e^z is taken as
// 2^(z log2 e).  CUDA's exp2f/expf add range handling that costs about 50
// cycles a call -- the bulk of a per-token softmax over 64 experts.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void latch_status(int32_t* status, int32_t code) {
    atomicCAS(status, 0, code);
}

// ---- bf16 / f32 element access ------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// relu, then round to bf16, of two floats in one instruction (PTX cvt .relu:
// a negative result becomes +0)
__device__ __forceinline__ uint32_t pack_relu_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.relu.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---- programmatic dependent launch ------------------------------------------
// The layer's kernels are launched with programmatic stream serialization: a
// kernel may be scheduled while its predecessor in the stream is finishing, so
// its prologue (barrier init, TMEM allocation, tensor-map prefetch) overlaps
// the predecessor's tail.  Every such kernel calls pdl_wait() before its first
// global-memory access (the predecessor has then completed: its writes are
// visible and its reads are done) and pdl_launch() right after, so a kernel's
// successor starts only once the kernel itself is past its own wait, and at
// most two kernels of the stream overlap.  Without the launch attribute both
// are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// false when MOE_B200_PDL=0 (plain stream order, kept for measurement)
bool pdl_enabled();

// Launch `kern` on stream s with programmatic stream serialization (unless
// disabled) and, for cluster_x > 1, clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_x,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// ---- per-device one-time settings ------------------------------------------
// Runs `set` once per (device, key); later calls return its first result.  key
// identifies the kernel instance (e.g. its address).  Thread-safe.
cudaError_t once_per_device(const void* key, cudaError_t (*set)(const void*));
// Number of SMs of the current device (cached).
cudaError_t device_sm_count(int* sms);

// ---- load-balancing loss from per-CTA router partials -------------------------
// "From Switch Transformer to GLaM", Load balancing: f_i = fraction of tokens
// whose top-1 choice is i, P_i = mean router probability of i, aux = alpha N
// sum_i f_i P_i.  part_cnt / part_psum hold, expert-major ([N][Gp], Gp = G
// rounded up to 4), each router CTA's top-1 counts and sums of p.  The sums run
// in fp64 in CTA order with a fixed partition over kAuxThreads threads, so every
// caller obtains the same bits.
struct AuxArgs {
    const int32_t* part_cnt; const float* part_psum;
    int G; int N; int64_t T; float alpha;   // G = 0: nothing to reduce
    double* f; double* P; double* aux;      // each nullable
    const double* part_z; double* z;        // router z-loss: per-CTA sums of lse^2 -> mean (z nullable)
};
constexpr int kAuxThreads = 192;
constexpr int kAuxScratch = 2 * kAuxThreads + 128;   // doubles of shared memory

// Router z-loss (CMU 10-423 Lecture 16, section 4.2, read as the mean over
// tokens of the squared log-sum-exp of the router logits) from per-CTA sums:
// called by one full warp; lane j adds partials j, j + 32, ... in order, then a
// fixed shuffle tree; z = total / T (0 for T = 0).
__device__ inline void z_reduce_warp(const double* part_z, int G, int64_t T, double* z) {
    const int lane = threadIdx.x & 31;
    double acc = 0.0;
    for (int g = lane; g < G; g += 32) acc += __ldcg(part_z + g);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) *z = T > 0 ? acc / (double)T : 0.0;
}

// Called by every thread of one block of at least kAuxThreads threads.
__device__ inline void aux_reduce_block(const AuxArgs& a, double* scratch) {
    const int tid = threadIdx.x;
    const int N = a.N, G = a.G, Gp = (G + 3) & ~3, nch = Gp / 4;
    const int tpe = kAuxThreads / N;   // threads per expert
    const int e = tid / tpe, j = tid % tpe;
    double* sp = scratch;
    double* sc = sp + kAuxThreads;
    double* sfp = sc + kAuxThreads;
    double pa = 0.0, ca = 0.0;
    if (tid < kAuxThreads && e < N) {   // this thread: chunks j, j + tpe, ... of 4 CTAs each, in order
        const float4* ps4 = reinterpret_cast<const float4*>(a.part_psum + (int64_t)e * Gp);
        const int4* cs4 = reinterpret_cast<const int4*>(a.part_cnt + (int64_t)e * Gp);
        for (int c0 = j; c0 < nch; c0 += 4 * tpe) {
            float4 pv[4];
            int4 cv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + u * tpe;
                pv[u] = c < nch ? __ldcg(ps4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                cv[u] = c < nch ? __ldcg(cs4 + c) : make_int4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int b = 4 * (c0 + u * tpe);   // first CTA of the chunk
                if (b + 0 < G) { pa += (double)pv[u].x; ca += (double)cv[u].x; }
                if (b + 1 < G) { pa += (double)pv[u].y; ca += (double)cv[u].y; }
                if (b + 2 < G) { pa += (double)pv[u].z; ca += (double)cv[u].z; }
                if (b + 3 < G) { pa += (double)pv[u].w; ca += (double)cv[u].w; }
            }
        }
    }
    if (tid < kAuxThreads) {
        sp[tid] = pa;
        sc[tid] = ca;
    }
    __syncthreads();
    if (tid < N) {
        double pt = 0.0, ct = 0.0;
        for (int q = 0; q < tpe; ++q) {
            pt += sp[tid * tpe + q];
            ct += sc[tid * tpe + q];
        }
        const double Pe = pt / (double)a.T, fe = ct / (double)a.T;
        if (a.P) a.P[tid] = Pe;
        if (a.f) a.f[tid] = fe;
        sfp[tid] = fe * Pe;
    }
    __syncthreads();
    if (tid == 0) {
        double s = 0.0;
        for (int q = 0; q < N; ++q) s += sfp[q];
        if (a.aux) *a.aux = (double)a.alpha * (double)N * s;
    }
    if (a.z && tid < 32) z_reduce_warp(a.part_z, G, a.T, a.z);
}

// ---- launchers implemented in the .cu files ---------------------------------
struct RouterArgs {
    const void* x; int dtype; const float* w_r; const float* b_r;
    int64_t T; int d; int N; int k;
    int32_t* idx; float* gate; float* probs;
    int32_t* part_cnt; float* part_psum;   // [nblk, N]
    double* f; double* P; double* aux; float alpha;
    double* part_z; double* z;             // router z-loss (z nullable; part_z [nblk] when z is set)
    void* w_split;                         // bf16 [3, NP, d] scratch (tensor-core router)
    int32_t* ticket;                       // finished-CTA counter of the tensor-core router
    int32_t* status;
    bool defer_aux;                        // tensor-core router: leave f, P, aux to aux_reduce_block
};
int router_tc_grid(int64_t T, int sms);            // CTAs of the tensor-core router (= partial rows used)

struct RouterBwdArgs {
    const void* x; int dtype; const float* w_r;
    const float* probs; const int32_t* idx; const float* gate; const double* f; const float* dgate;
    float alpha; int64_t T; int d; int N; int k;
    float* dh;                        // [T, N]
    float* dw; float* db; float* dx;  // [N, d], [N], [T, d] (each nullable)
    float* part_dw; float* part_db;   // [router_bwd_chunks(T), N, d], [.., N]
    // tensor-core path (bf16 x): workspace regions, see router_bwd_tc_bytes
    void* tc_adx; void* tc_adw; void* tc_bdx; int32_t* tc_offs; float* tc_part;
    int32_t* status;
};
int router_bwd_chunks(int64_t T);
// tensor-core router backward: padded experts (a multiple of 16), tokens per
// dW_r chunk (at most 128 chunks), and the chunk count
int router_bwd_np16(int N);
int64_t router_bwd_tc_chunk(int64_t T);
int router_bwd_tc_chunks(int64_t T);
cudaError_t launch_router_backward(const RouterBwdArgs& a, cudaStream_t s);
int router_blocks(int64_t T, int N);               // partial rows the FP32-pipe router writes
int router_partial_rows(int64_t T, int N);         // partial rows any router path writes
int router_tc_padded_experts(int N);
cudaError_t launch_router(const RouterArgs& a, cudaStream_t s);
cudaError_t launch_router_tc(const RouterArgs& a, cudaStream_t s);
cudaError_t launch_aux_finalize(const double* part_z, double* z, const int32_t* part_cnt, const float* part_psum,
                                int nblk, int N, int64_t T,
                                float alpha, double* f, double* P, double* aux, cudaStream_t s);

// Number of claims numbered base, base+1, ..., base+count-1 that fall below C.
__host__ __device__ __forceinline__ int kept_after(int base, int count, int C) {
    const int room = C - base;
    return room <= 0 ? 0 : (room < count ? room : count);
}

// Batch-priority scratch (all device, workspace-held); perm == nullptr: token order.
constexpr int kPrioBuckets = 1 << 16;
struct PrioArgs {
    int32_t* hist;        // [kPrioBuckets + 1] bucket counts, then their exclusive prefix
    int32_t* cursor;      // [kPrioBuckets]
    int32_t* list;        // [T] tokens grouped by bucket
    int32_t* perm;        // [T] perm[place] = token
    int32_t* idx_sorted;  // [T, k] expert choices in claim order
    int32_t* pos_sorted;  // [T, k] claim numbers in claim order
    uint32_t* range;      // [2] smallest and largest key of the batch
};

struct DispatchArgs {
    const void* x; int dtype; const int32_t* idx; const float* gate;
    int64_t T; int d; int N; int k; int C;
    int32_t* pos; uint8_t* drop; int32_t* counts; int32_t* kept; int32_t* offsets;
    int32_t* row_token; float* row_gate; void* xe;
    void* zero_out;              // top-1 fused path: rows of dropped tokens are zeroed
    uint32_t* scan_state; WsHeader* hdr;
    const int32_t* claim_base;   // [k, N] claims made before this shard (sharded batch), or null
    AuxArgs aux;                 // G > 0: one extra block of the gather reduces the router partials
    PrioArgs prio;               // batch priority (perm set) or token order
};
// No-Token-Left-Behind re-routing (top-1); all device, workspace-held scratch.
struct NtlbArgs {
    const void* x; int dtype; const float* probs;   // probs [T, N]
    int64_t T; int d; int N; int C;
    int32_t* expert; float* gate; int32_t* pos; uint8_t* drop;   // [T], token order
    int32_t* counts; int32_t* kept; int32_t* offsets;            // [N], [N], [N + 1]
    int32_t* row_token; float* row_gate; void* xe; void* zero_out;
    int32_t* ch; int32_t* last; int32_t* first; int32_t* placed; int32_t* lp;   // [T] each
    int32_t* grid_agg;        // [2][kNtlbMaxBlocks][N] per-block stage claims
    int32_t* grid_unplaced;   // [2][kNtlbMaxBlocks]
    uint32_t* grid_bar;       // grid barrier counter
    WsHeader* hdr;
    AuxArgs aux;
};
constexpr int kNtlbMaxBlocks = 256;   // blocks of the cooperative re-routing kernel
cudaError_t launch_dispatch_ntlb(const NtlbArgs& a, cudaStream_t s);

int scan_blocks(int64_t T);
cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s);
cudaError_t launch_counts(const int32_t* idx, int64_t T, int N, int k, int32_t* counts, cudaStream_t s);
cudaError_t launch_claim_base(const int32_t* all, int S, int shard, int k, int N, int32_t* base, cudaStream_t s);
cudaError_t launch_aux_shards(int S, int N, const int64_t* tokens, const double* f_all, const double* P_all,
                              float alpha, double* f, double* P, double* aux, cudaStream_t s);
cudaError_t launch_lookback_timeout_probe(uint32_t* state, WsHeader* hdr, long long limit_ns,
                                          cudaStream_t s);

struct FfnArgs {
    int dtype; int act; int N; int d; int d_ff; int C; int64_t R_cap;
    const void* xe; const int32_t* offsets;
    const void* w1; const void* b1; const void* w3; const void* b3;
    const void* w2; const void* b2;
    void* h;                      // [R_cap, d_ff] scratch
    void* ye;                     // [R, d] (used when scatter_out == nullptr)
    void* scatter_out;            // top-1 fused: out[row_token[r]] = row_gate[r] * E(x)
    const int32_t* row_token; const float* row_gate;
    // expert parallelism: row r's result goes to GPU row_rank[r]: scatter_ptrs
    // [row_rank[r]] + row_token[r] * d, times row_gate[r] (nullable: 1)
    void* const* scatter_ptrs; const int32_t* row_rank;
    WsHeader* hdr;
    void* mid_event;              // optional cudaEvent_t recorded between the two stages
    void* pre_out;                // SwiGLU (optional): stage-1 pre-activations [R, 2 d_ff]
    bool stage1_only;             // the first GEMM only (the backward's recompute)
};
cudaError_t launch_expert_ffn(const FfnArgs& a, cudaStream_t s);
cudaError_t launch_expert_ffn_tc(const FfnArgs& a, cudaStream_t s);

// Expert FFN backward on the tensor cores (gemm_bwd.cu), bf16.
struct BwdArgs {
    int act; int N; int d; int d_ff; int k; int64_t T; int64_t R_cap;
    const void* xe; const int32_t* offsets; const int32_t* row_token; const float* row_gate;
    const int32_t* idx; const int32_t* pos; const uint8_t* drop;
    const void* dout;
    const void* w1; const void* b1; const void* w3; const void* b3; const void* w2;
    float* dx; float* dw1; float* db1; float* dw3; float* db3; float* dw2; float* db2;
    bool top1_scatter;            // dx rows scattered by token (top-1), else combined from dxe
    void* h; void* pre; void* dy; void* du; float* dxe;   // workspace
    WsHeader* hdr;
};
cudaError_t launch_expert_backward_tc(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_tc_rows_f32(const void* A, int64_t rows, int K, const void* B, int n, const int32_t* offsets,
                               float* out, int32_t* status, cudaStream_t s);
cudaError_t launch_tc_weights_f32(const void* A, int64_t rows, int m, const void* B, int n, const int32_t* offsets,
                                  int groups, float* out, int32_t* status, cudaStream_t s);

// Expert parallelism (ep.cu)
struct EpDispatchArgs {
    int dtype; int64_t T; int d; int N; int k; int G; int rank; int64_t R_cap;
    const void* x; const int32_t* offsets; const int32_t* row_token; const float* row_gate;
    const int32_t* dst_start; const uint8_t* drop; void* out;
    void* const* recv_x; int32_t* const* recv_rank; int32_t* const* recv_row; float* const* recv_gate;
};
cudaError_t launch_ep_layout(int G, int rank, int N, const int32_t* kept_all, int32_t* dst_start,
                             int32_t* recv_offsets, cudaStream_t s);
cudaError_t launch_ep_dispatch(const EpDispatchArgs& a, cudaStream_t s);
cudaError_t launch_ep_return(int dtype, const void* ye, const int32_t* recv_offsets, int E, int d, int64_t R_cap,
                             const int32_t* recv_rank, const int32_t* recv_row, const float* recv_gate,
                             void* const* out_ptrs, cudaStream_t s);

struct CombineArgs {
    int dtype; int64_t T; int d; int k;
    const void* ye; const int32_t* idx; const int32_t* pos; const uint8_t* drop;
    const float* gate; const int32_t* offsets; void* out;
    // one shard of a routing group (both null otherwise): pos are group-wide
    // claim numbers; claim_base [k, N] and the shard's own counts [k, N] map
    // them to the shard's rows.  C is the group capacity.
    const int32_t* claim_base; const int32_t* counts; int C; int N;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

struct GateGradArgs {
    int dtype; int64_t T; int d; int k;
    const void* dout; const void* ye; const int32_t* idx; const int32_t* pos; const uint8_t* drop;
    const int32_t* offsets; float* dgate;
};
cudaError_t launch_gate_grad(const GateGradArgs& a, cudaStream_t s);

}  // namespace moe
