// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every expert e and every compact row of e (rows
// [offsets[e], offsets[e+1]) of A):
//   stage 1, ReLU   : H = relu(A W1[e]^T + b1[e])
//   stage 1, SwiGLU : H = silu(A W1[e]^T + b1[e]) * (A W3[e]^T + b3[e])
//   stage 2         : Y = H W2[e]^T + b2[e]            (compact rows), or
//   stage 2, scatter: out[row_token[r]] = row_gate[r] * (H W2[e]^T + b2[e])[r]
// which is the expert FFN of "From Switch Transformer to GLaM" (FFN(x) =
// W2 s(W1 x)), the Mixtral SwiGLU expert of CMU 10-423 Lecture 16 section 2.3,
// and the gate-scaled top-1 combine y = p_{i*} E_{i*}(x) of the GLaM page.
//
// Kernel design (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 0   TMA producer: 128x64 A tile + 256x64 B tile per stage (128-byte
//            swizzle, 4-stage mbarrier ring).  For SwiGLU the 256 B rows are 128
//            rows of W1 followed by the same 128 rows of W3, so ONE N=256 MMA
//            produces the gate and up halves side by side in TMEM.
//   warp 1   TMEM allocator + MMA issuer: tcgen05.mma.cta_group::1.kind::f16,
//            M=128 N=256 K=16, bf16 x bf16 -> fp32 in TMEM; two 256-column
//            accumulators (all 512 columns) so the epilogue of tile i overlaps
//            the main loop of tile i+1.
//   warps 2-5 epilogue: tcgen05.ld 32x32b (thread = row), bias, activation,
//            gate, bf16 pack, 16-byte stores (optionally scattered to token rows).
// Tiles: an expert's rows are cut into 128-row m-tiles; the tile list is
// expert-major with m-tiles grouped by 8 inside an expert (concurrent CTAs share
// B columns and A rows in L2).  Rows past an expert's end inside its last m-tile
// belong to the next expert (or are zero-filled out of bounds); the MMA computes
// them and the epilogue masks them.
// Every wait on an mbarrier is bounded: on expiry the kernel latches
// MOE_ERR_TIMEOUT, stops issuing work, waits (bounded) for its own copies and
// MMAs in flight, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;          // MMA N (and TMEM columns per accumulator)
constexpr int BK = 64;           // 64 bf16 = one 128-byte swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
constexpr int TMEM_COLS = 512;
constexpr int GEMM_THREADS = 192;
constexpr int GROUP_M = 8;

enum { EPI_RELU = 0, EPI_SWIGLU = 1, EPI_BIAS = 2, EPI_SCATTER = 3 };

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (7-9 = 1),
// B bf16 (10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct GemmParams {
    const int32_t* offsets;   // [N + 1] compact row ranges
    int N;
    int n_dim;                // output columns per expert
    int k_dim;                // reduction length
    int out_ld;
    const __nv_bfloat16* bias;
    const __nv_bfloat16* bias3;
    __nv_bfloat16* out;
    const int32_t* row_token;
    const float* row_gate;
    int32_t* status;
    long long limit_ns;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

struct Waiter {
    volatile int* abort;
    int32_t* status;
    long long limit;
};

// Bounded wait for the phase of the given parity.  Gives up when another role
// has aborted, or after `limit` ns (then it latches MOE_ERR_TIMEOUT and aborts).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Waiter& w) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 255u) == 0u) {
            if (*w.abort) return false;
            if (global_ns() - t0 > w.limit) {
                *w.abort = 1;
                latch_status(w.status, MOE_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Teardown wait: ignores the abort flag, still bounded.
__device__ __forceinline__ bool drain_bar(uint32_t bar, uint32_t parity, long long limit, int32_t* status) {
    const long long t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 255u) == 255u && global_ns() - t0 > limit) {
            latch_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
          "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
          "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
          "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct TileInfo {
    int e, row0, rows, n0;
};

// tile -> (expert, first compact row, valid rows, first output column)
__device__ __forceinline__ TileInfo decode_tile(int tile, const int* prefix, const int* off, int N, int ntn,
                                                int bn_out) {
    int lo = 0, hi = N;   // prefix[lo] <= tile < prefix[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (prefix[mid] <= tile) lo = mid;
        else hi = mid;
    }
    const int e = lo;
    const int rows_e = off[e + 1] - off[e];
    const int mt = (rows_e + BM - 1) / BM;
    const int local = tile - prefix[e];
    const int per_group = GROUP_M * ntn;
    const int g = local / per_group;
    const int first_m = g * GROUP_M;
    const int gsz = min(mt - first_m, GROUP_M);
    const int rem = local - g * per_group;
    const int m_blk = first_m + rem % gsz;
    const int n_blk = rem / gsz;
    TileInfo ti;
    ti.e = e;
    ti.row0 = off[e] + m_blk * BM;
    ti.rows = min(BM, rows_e - m_blk * BM);
    ti.n0 = n_blk * bn_out;
    return ti;
}

__device__ __forceinline__ float silu(float z) { return z / (1.f + expf(-z)); }

template <int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB3, const GemmParams p) {
    constexpr int BN_OUT = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[STAGES];
    __shared__ __align__(8) uint64_t empty_bar[STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_off[129];
    __shared__ int s_prefix[129];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N;
    for (int i = tid; i <= N; i += GEMM_THREADS) s_off[i] = p.offsets[i];
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull_bar[a]), 1);
            mbar_init(smem_u32(&tempty_bar[a]), 128);
        }
        mbar_init(smem_u32(&done_bar), 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    const int ntn = (p.n_dim + BN_OUT - 1) / BN_OUT;
    if (tid == 0) {
        int acc = 0;
        for (int e = 0; e < N; ++e) {
            s_prefix[e] = acc;
            acc += ((s_off[e + 1] - s_off[e] + BM - 1) / BM) * ntn;
        }
        s_prefix[N] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = s_tmem;
    const int total = s_prefix[N];
    const int nkb = (p.k_dim + BK - 1) / BK;
    const Waiter w{&s_abort, p.status, p.limit_ns};

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int last_par[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) last_par[s] = -1;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, s_prefix, s_off, N, ntn, BN_OUT);
                const int brow = ti.e * p.n_dim + ti.n0;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(smem_u32(&empty_bar[stage]), phase ^ 1u, w)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t a_dst = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t b_dst = a_dst + A_BYTES;
                    mbar_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(a_dst, &tmA, fb, kb * BK, ti.row0);
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(b_dst, &tmB, fb, kb * BK, brow);
                        tma_load_2d(b_dst + B_BYTES / 2, &tmB3, fb, kb * BK, brow);
                    } else {
                        tma_load_2d(b_dst, &tmB, fb, kb * BK, brow);
                    }
                    last_par[stage] = (int)phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every load this thread issued has landed before the CTA retires
            for (int s = 0; s < STAGES; ++s)
                if (last_par[s] >= 0) drain_bar(smem_u32(&full_bar[s]), (uint32_t)last_par[s], p.limit_ns, p.status);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
                if (!wait_bar(smem_u32(&tempty_bar[acc]), acc_par ^ 1u, w)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(smem_u32(&full_bar[stage]), phase, w)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issued = true;
                    const uint32_t a_addr = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        umma_f16(d_tmem, umma_desc(a_addr + kk * 32), umma_desc(b_addr + kk * 32), kIdesc,
                                 (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&empty_bar[stage]));   // frees the stage when these MMAs finish
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit(smem_u32(&tfull_bar[acc]));
            }
            // all MMAs issued by this thread have completed before TMEM is freed
            if (issued) {
                umma_commit(smem_u32(&done_bar));
                drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int r_in_tile = q * 32 + lane;
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            const TileInfo ti = decode_tile(tile, s_prefix, s_off, N, ntn, BN_OUT);
            const int acc = it & 1;
            const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
            const bool got = wait_bar(smem_u32(&tfull_bar[acc]), acc_par, w);
            if (!__all_sync(0xffffffffu, got)) break;   // warp-uniform exit on abort
            tc_fence_after();
            const bool valid = r_in_tile < ti.rows;
            const int64_t grow = (int64_t)ti.row0 + r_in_tile;
            int64_t orow = grow;
            float g = 1.f;
            if (EPI == EPI_SCATTER && valid) {
                orow = p.row_token[grow];
                g = p.row_gate[grow];
            }
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const __nv_bfloat16* bias_e = p.bias ? p.bias + (int64_t)ti.e * p.n_dim : nullptr;
            const __nv_bfloat16* bias3_e = p.bias3 ? p.bias3 + (int64_t)ti.e * p.n_dim : nullptr;
            __nv_bfloat16* out_row = p.out + orow * (int64_t)p.out_ld;
#pragma unroll 1
            for (int c = 0; c < BN_OUT / 32; ++c) {
                uint32_t u[32];
                tmem_ld32(tbase + c * 32, u);
                uint32_t v[32];
                if (EPI == EPI_SWIGLU) tmem_ld32(tbase + BN_OUT + c * 32, v);
                tmem_wait_ld();
                const int col = ti.n0 + c * 32;
                if (valid && col < p.n_dim) {
                    float bu[32], bv[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        bu[j] = 0.f;
                        bv[j] = 0.f;
                    }
                    if (bias_e) {
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            if (col + 8 * g8 < p.n_dim) {
                                uint4 bw = __ldg(reinterpret_cast<const uint4*>(bias_e + col + 8 * g8));
                                const uint32_t* bp = reinterpret_cast<const uint32_t*>(&bw);
#pragma unroll
                                for (int h = 0; h < 4; ++h) {
                                    bu[8 * g8 + 2 * h] = bf16lo(bp[h]);
                                    bu[8 * g8 + 2 * h + 1] = bf16hi(bp[h]);
                                }
                            }
                        }
                    }
                    if (EPI == EPI_SWIGLU && bias3_e) {
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            if (col + 8 * g8 < p.n_dim) {
                                uint4 bw = __ldg(reinterpret_cast<const uint4*>(bias3_e + col + 8 * g8));
                                const uint32_t* bp = reinterpret_cast<const uint32_t*>(&bw);
#pragma unroll
                                for (int h = 0; h < 4; ++h) {
                                    bv[8 * g8 + 2 * h] = bf16lo(bp[h]);
                                    bv[8 * g8 + 2 * h + 1] = bf16hi(bp[h]);
                                }
                            }
                        }
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float a0 = __uint_as_float(u[2 * j]) + bu[2 * j];
                        float a1 = __uint_as_float(u[2 * j + 1]) + bu[2 * j + 1];
                        if (EPI == EPI_RELU) {
                            a0 = fmaxf(a0, 0.f);
                            a1 = fmaxf(a1, 0.f);
                        } else if (EPI == EPI_SWIGLU) {
                            a0 = silu(a0) * (__uint_as_float(v[2 * j]) + bv[2 * j]);
                            a1 = silu(a1) * (__uint_as_float(v[2 * j + 1]) + bv[2 * j + 1]);
                        } else if (EPI == EPI_SCATTER) {
                            a0 *= g;
                            a1 *= g;
                        }
                        packed[j] = pack_bf16x2(a0, a1);
                    }
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        if (col + 8 * g8 < p.n_dim) {
                            *reinterpret_cast<uint4*>(out_row + col + 8 * g8) =
                                make_uint4(packed[4 * g8], packed[4 * g8 + 1], packed[4 * g8 + 2], packed[4 * g8 + 3]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty_bar[acc]));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------- host ----

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
    static EncodeFn fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeFn) nullptr;
        return reinterpret_cast<EncodeFn>(ptr);
    }();
    return fn;
}

// 2-D bf16 tensor [rows, k] (k contiguous), box = box_rows x 64, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t k, int box_rows) {
    EncodeFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)k * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sms = 0;
    bool attr_set[4] = {false, false, false, false};
};
std::mutex g_mu;
DeviceInfo g_dev[64];

template <int EPI>
cudaError_t run_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b3, const GemmParams& p,
                     cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    int sms;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        DeviceInfo& di = g_dev[dev & 63];
        if (di.sms == 0) {
            err = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
        }
        if (!di.attr_set[EPI]) {
            err = cudaFuncSetAttribute(grouped_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
            if (err != cudaSuccess) return err;
            di.attr_set[EPI] = true;
        }
        sms = di.sms;
    }
    grouped_gemm_kernel<EPI><<<sms, GEMM_THREADS, SMEM_BYTES, s>>>(a, b, b3, p);
    return cudaGetLastError();
}

}  // namespace

// Stage 1 + stage 2 of the bf16 expert FFN on the tensor cores.
cudaError_t launch_expert_ffn_tc(const FfnArgs& a, cudaStream_t s) {
    const int64_t R = a.R_cap > 0 ? a.R_cap : 1;
    CUtensorMap mA1, mB1, mB3, mA2, mB2;
    const bool swiglu = a.act == MOE_SWIGLU;
    if (!make_map(&mA1, a.xe, R, a.d, BM) || !make_map(&mB1, a.w1, (int64_t)a.N * a.d_ff, a.d, swiglu ? BN / 2 : BN) ||
        !make_map(&mA2, a.h, R, a.d_ff, BM) || !make_map(&mB2, a.w2, (int64_t)a.N * a.d, a.d_ff, BN))
        return cudaErrorInvalidValue;
    if (swiglu) {
        if (!make_map(&mB3, a.w3, (int64_t)a.N * a.d_ff, a.d, BN / 2)) return cudaErrorInvalidValue;
    } else {
        mB3 = mB1;
    }
    GemmParams p1{};
    p1.offsets = a.offsets;
    p1.N = a.N;
    p1.n_dim = a.d_ff;
    p1.k_dim = a.d;
    p1.out_ld = a.d_ff;
    p1.bias = reinterpret_cast<const __nv_bfloat16*>(a.b1);
    p1.bias3 = reinterpret_cast<const __nv_bfloat16*>(a.b3);
    p1.out = reinterpret_cast<__nv_bfloat16*>(a.h);
    p1.status = &a.hdr->status;
    p1.limit_ns = kWaitLimitNs;
    cudaError_t err = swiglu ? run_gemm<EPI_SWIGLU>(mA1, mB1, mB3, p1, s) : run_gemm<EPI_RELU>(mA1, mB1, mB3, p1, s);
    if (err != cudaSuccess) return err;
    if (a.mid_event && (err = cudaEventRecord((cudaEvent_t)a.mid_event, s)) != cudaSuccess) return err;

    GemmParams p2{};
    p2.offsets = a.offsets;
    p2.N = a.N;
    p2.n_dim = a.d;
    p2.k_dim = a.d_ff;
    p2.out_ld = a.d;
    p2.bias = reinterpret_cast<const __nv_bfloat16*>(a.b2);
    p2.status = &a.hdr->status;
    p2.limit_ns = kWaitLimitNs;
    if (a.scatter_out) {
        p2.out = reinterpret_cast<__nv_bfloat16*>(a.scatter_out);
        p2.row_token = a.row_token;
        p2.row_gate = a.row_gate;
        return run_gemm<EPI_SCATTER>(mA2, mB2, mB2, p2, s);
    }
    p2.out = reinterpret_cast<__nv_bfloat16*>(a.ye);
    return run_gemm<EPI_BIAS>(mA2, mB2, mB2, p2, s);
}

}  // namespace moe
