// Backward of the expert FFN on the 5th-generation tensor cores.
//
// Forward, per kept assignment (row r of expert e, token t, gate g):
//   u = W1[e] x + b1,  a = relu(u)   (SwiGLU: a = silu(W1 x + b1) * (W3 x + b3)),
//   y = W2[e] a + b2,  out_t += g y
// ("From Switch Transformer to GLaM", FFN(x) = W2 s(W1 x); CMU 10-423 Lecture
// 16, section 2.3, the Mixtral SwiGLU expert).  With dY[r] = g dL/dout_t:
//   dA  = dY W2[e]                       (row GEMM, B = W2 read MN-major)
//   dU  = dA * relu'(u)                   (SwiGLU: dG = dA * up * silu'(gate_pre),
//                                          dUp = dA * silu(gate_pre))
//   dx_t += dU W1[e]  (+ dUp W3[e])       (row GEMM, B = W1 / W3 read MN-major)
//   dW1[e] = dU^T X_e,  dW3[e] = dUp^T X_e,  dW2[e] = dY^T A_e
//                                         (weight GEMMs: the reduction runs
//                                          over the expert's rows, both operands
//                                          read MN-major)
//   db1 = column sums of dU, db3 of dUp, db2 of dY.
//
// One kernel template, single CTA per tile (M = 128, N = 256), persistent,
// warp-specialised like the forward GEMM: warp 0 TMA producer, warp 1 MMA
// issuer (and, in the weight GEMMs, the warp that zeroes the rows of a K block
// past the expert's last row, since those rows belong to the next expert),
// warps 2-5 epilogue.  Operands:
//   K-major A (row GEMMs): box 64 K x 128 rows, as in the forward;
//   MN-major A / B: boxes of 64 MN elements x 64 K rows (128-byte swizzle), two
//   for A (M = 128), four for B (N = 256), 8 KB apart -- one blocked 3-D TMA
//   load each when the matrix's columns are a multiple of 64.
// Epilogues: fp32 outputs (dW, compact dx) and the ReLU dU leave through
// swizzled shared-memory staging rows and TMA tensor stores; scattered dx rows
// as 128-byte row pieces; the dU epilogue loads its forward values (H or the
// SwiGLU pre-activations) one 32-column chunk ahead.
// Every mbarrier wait is bounded (MOE_ERR_TIMEOUT on expiry, then a bounded
// drain of the copies and MMAs in flight before TMEM is freed).
#include "tc_common.cuh"

namespace moe {
using namespace tc;
namespace {

constexpr int BW_BM = 128, BW_BN = 256, BW_BK = 64;
constexpr int BW_THREADS = 192;
constexpr int BW_STAGES = 4;
constexpr int BW_A_BYTES = BW_BM * BW_BK * 2;   // 16 KB
constexpr int BW_B_BYTES = BW_BN * BW_BK * 2;   // 32 KB
constexpr int BW_STAGE_BYTES = BW_A_BYTES + BW_B_BYTES;
// fp32 epilogues (weight gradients, dx): per epilogue warp two staging buffers
// of 32 rows x 128 bytes (32 fp32 columns), written out with TMA tensor stores
constexpr int BW_EPI_BYTES = 4 * 2 * 32 * 128;
constexpr int BW_SMEM = BW_STAGES * BW_STAGE_BYTES + BW_EPI_BYTES + 1024;
static_assert((BW_STAGES * BW_STAGE_BYTES) % 1024 == 0, "staging buffers 1024-byte aligned");
constexpr int BW_TMEM_COLS = 512;
constexpr int MN_BOX = 64 * BW_BK * 2;          // one MN-major box: 64 MN x 64 K rows = 8 KB

enum { BW_DU_RELU = 0, BW_DU_SWIGLU = 1, BW_DX = 2, BW_WGT = 3 };

struct BwdParams {
    const int32_t* offsets;   // [N + 1] compact rows of each expert
    int N;
    int m_dim, n_dim, k_dim;  // weight GEMMs: M, N per expert (K = its rows); row GEMMs: N, K
    int k_split;              // row GEMM with two B tensors: K blocks below k_split read B, above B2
    // epilogues
    const __nv_bfloat16* h;   // BW_DU_RELU: H [R, n_dim] (relu'(u) = H > 0)
    const __nv_bfloat16* pre; // BW_DU_SWIGLU: gate and up pre-activations [R, 2 n_dim]
    __nv_bfloat16* du;        // BW_DU_*: dU [R, n_dim] or dG | dUp [R, 2 n_dim]
    float* out;               // BW_DX: dx rows (scatter: [T, n_dim] by row_token; else [R, n_dim]);
                              // BW_WGT: dW [N, m_dim, n_dim]
    const int32_t* row_token; // BW_DX scatter (top-1)
    int mn3;                  // bit 0: tmA is a blocked 3-D MN map (2 blocks per load),
                              // bit 1: tmB and tmB2 are (4 blocks per load)
    int32_t* status;
    long long limit_ns;
};

struct BwTile {
    int e, row0, rows, m0, n0, k_rows, k_row0;
};

template <int MODE>
__device__ __forceinline__ BwTile bw_decode(int tile, const int* prefix, const int* off, int N, int ntm, int ntn) {
    BwTile t{};
    if (MODE == BW_WGT) {   // (expert, m-tile, n-tile) over every expert, n fastest
        const int per_e = ntm * ntn;
        t.e = tile / per_e;
        const int rem = tile - t.e * per_e;
        t.m0 = (rem / ntn) * BW_BM;
        t.n0 = (rem % ntn) * BW_BN;
        t.k_row0 = off[t.e];
        t.k_rows = off[t.e + 1] - off[t.e];
        return t;
    }
    int lo = 0, hi = N;   // prefix[lo] <= tile < prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= tile) lo = mid;
        else hi = mid;
    }
    t.e = lo;
    const int local = tile - prefix[lo];
    const int m_blk = local / ntn;
    t.n0 = (local - m_blk * ntn) * BW_BN;
    t.row0 = off[lo] + m_blk * BW_BM;
    t.rows = min(BW_BM, off[lo + 1] - t.row0);
    return t;
}

__device__ __forceinline__ float sigmoidf_(float z) { return __fdividef(1.f, 1.f + fast_exp2(-z * kLog2e)); }

template <int MODE>
__global__ void __launch_bounds__(BW_THREADS, 1)
bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmOut,
                const BwdParams p) {
    constexpr bool A_MN = MODE == BW_WGT;
    constexpr uint32_t IDESC = idesc_bf16_f32_major(BW_BM, BW_BN, A_MN, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[BW_STAGES];
    __shared__ __align__(8) uint64_t empty_bar[BW_STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_off[129];
    __shared__ int s_prefix[129];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N;
    if (tid == 0) {
        for (int s = 0; s < BW_STAGES; ++s) {
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
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) tmem_alloc(&s_tmem, BW_TMEM_COLS);
    pdl_wait();
    pdl_launch();
    for (int i = tid; i <= N; i += BW_THREADS) s_off[i] = p.offsets[i];
    __syncthreads();
    const int ntn = (p.n_dim + BW_BN - 1) / BW_BN;
    const int ntm = (p.m_dim + BW_BM - 1) / BW_BM;
    if (warp == 2) {
        if (MODE == BW_WGT) {
            if (lane == 0) s_prefix[N] = N * ntm * ntn;
        } else {   // tiles per expert (128-row m-tiles x n-tiles) and their exclusive prefix
            int cnt[4], sum = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = lane * 4 + j;
                cnt[j] = e < N ? ((s_off[e + 1] - s_off[e] + BW_BM - 1) / BW_BM) * ntn : 0;
                sum += cnt[j];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int run = incl - sum;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = lane * 4 + j;
                if (e < N) s_prefix[e] = run;
                run += cnt[j];
            }
            if (lane == 31) s_prefix[N] = incl;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = s_tmem;
    const int total = s_prefix[N];
    const Waiter w{&s_abort, p.status, p.limit_ns};
    auto nkb_of = [&](const BwTile& ti) {
        return MODE == BW_WGT ? (ti.k_rows + BW_BK - 1) / BW_BK : (p.k_dim + BW_BK - 1) / BW_BK;
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int last_par[BW_STAGES];
#pragma unroll
            for (int s = 0; s < BW_STAGES; ++s) last_par[s] = -1;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const BwTile ti = bw_decode<MODE>(tile, s_prefix, s_off, N, ntm, ntn);
                const int nkb = nkb_of(ti);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(smem_u32(&empty_bar[stage]), phase ^ 1u, w)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t a_dst = smem_u32(smem + stage * BW_STAGE_BYTES);
                    const uint32_t b_dst = a_dst + BW_A_BYTES;
                    mbar_expect_tx(fb, BW_STAGE_BYTES);
                    if (MODE == BW_WGT) {
                        const int kr = ti.k_row0 + kb * BW_BK;   // rows of the expert (K)
                        if (p.mn3 & 1) {
                            tma_load_3d(a_dst, &tmA, fb, 0, kr, ti.m0 / 64);
                        } else {
#pragma unroll
                            for (int j = 0; j < 2; ++j) tma_load_2d(a_dst + j * MN_BOX, &tmA, fb, ti.m0 + 64 * j, kr);
                        }
                        if (p.mn3 & 2) {
                            tma_load_3d(b_dst, &tmB, fb, 0, kr, ti.n0 / 64);
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) tma_load_2d(b_dst + j * MN_BOX, &tmB, fb, ti.n0 + 64 * j, kr);
                        }
                    } else {
                        tma_load_2d(a_dst, &tmA, fb, kb * BW_BK, ti.row0);
                        // B = weights [N_exp * K rows][n cols]; two tensors split at k_split
                        const bool second = p.k_split > 0 && kb * BW_BK >= p.k_split;
                        const int kk = second ? kb * BW_BK - p.k_split : kb * BW_BK;
                        const int kdim_b = p.k_split > 0 ? p.k_split : p.k_dim;
                        const CUtensorMap* bm = second ? &tmB2 : &tmB;
                        if (p.mn3 & 2) {
                            tma_load_3d(b_dst, bm, fb, 0, ti.e * kdim_b + kk, ti.n0 / 64);
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                tma_load_2d(b_dst + j * MN_BOX, bm, fb, ti.n0 + 64 * j, ti.e * kdim_b + kk);
                        }
                    }
                    last_par[stage] = (int)phase;
                    if (++stage == BW_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < BW_STAGES; ++s)
                if (last_par[s] >= 0) drain_bar(smem_u32(&full_bar[s]), (uint32_t)last_par[s], p.limit_ns, p.status);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (lane 0); the warp zeroes K rows past an expert's end ----------------
        int stage = 0;
        uint32_t phase = 0;
        int it = 0;
        bool ok = true, issued = false;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
            const BwTile ti = bw_decode<MODE>(tile, s_prefix, s_off, N, ntm, ntn);
            const int nkb = nkb_of(ti);
            const int acc = it & 1;
            const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
            bool got = wait_bar(smem_u32(&tempty_bar[acc]), acc_par ^ 1u, w);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BW_BN);
            for (int kb = 0; kb < nkb; ++kb) {
                got = wait_bar(smem_u32(&full_bar[stage]), phase, w);   // every lane: the copies have landed
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + stage * BW_STAGE_BYTES);
                const uint32_t b_addr = a_addr + BW_A_BYTES;
                if (MODE == BW_WGT) {
                    const int valid = ti.k_rows - kb * BW_BK;   // K rows of this block that are the expert's
                    if (valid < BW_BK) {
                        // rows [valid, 64) of each box: the next expert's rows (or out of bounds)
                        uint8_t* st = smem + stage * BW_STAGE_BYTES;
                        const int nz = (BW_BK - valid) * 128 / 16;   // 16-byte words per box
                        for (int bx = 0; bx < 6; ++bx) {
                            uint4* z = reinterpret_cast<uint4*>(st + bx * MN_BOX + valid * 128);
                            for (int q = lane; q < nz; q += 32) z[q] = make_uint4(0, 0, 0, 0);
                        }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                    }
                }
                if (lane == 0) {
                    issued = true;
                    // the next 16-deep K slice: +32 bytes in a K-major tile, +16 rows of
                    // 128 bytes in an MN-major one (the address field counts 16 bytes)
                    const uint64_t ad0 = A_MN ? umma_desc_mn(a_addr, MN_BOX) : umma_desc(a_addr);
                    const uint64_t bd0 = umma_desc_mn(b_addr, MN_BOX);
#pragma unroll
                    for (int kk = 0; kk < BW_BK / 16; ++kk) {
                        const uint64_t ad = ad0 + (uint64_t)(kk * (A_MN ? 2048 / 16 : 32 / 16));
                        const uint64_t bd = bd0 + (uint64_t)(kk * (2048 / 16));
                        umma_f16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&empty_bar[stage]));
                }
                __syncwarp();
                if (++stage == BW_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // no K block (an expert without rows): the accumulator is never written, and
            // the epilogue writes zeros; the commit still orders the hand-over
            if (ok && lane == 0) umma_commit(smem_u32(&tfull_bar[acc]));
            __syncwarp();
        }
        if (lane == 0) {
            umma_commit(smem_u32(&done_bar));
            drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
        }
        (void)issued;
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 2..5): thread = accumulator row ----------------
        const int q = warp & 3;
        const int r_in = q * 32 + lane;
        const uint32_t ebuf0 = smem_u32(smem + BW_STAGES * BW_STAGE_BYTES + q * 2 * 32 * 128);
        uint32_t nchunk = 0;   // chunks staged so far (buffer = nchunk & 1; one bulk group each)
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            const BwTile ti = bw_decode<MODE>(tile, s_prefix, s_off, N, ntm, ntn);
            const int acc = it & 1;
            const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
            // dU epilogues read this row's forward values (H, or the SwiGLU
            // pre-activations) for each 32-column chunk: they are loaded one chunk
            // ahead (the first before the accumulator wait), so the global-load
            // latency overlaps the previous chunk instead of stalling every chunk
            constexpr bool DU = MODE == BW_DU_RELU || MODE == BW_DU_SWIGLU;
            constexpr int NPF = MODE == BW_DU_SWIGLU ? 8 : (MODE == BW_DU_RELU ? 4 : 1);   // 16-byte loads per chunk
            const bool row_ok = DU && r_in < ti.rows;
            const int64_t r_du = (int64_t)ti.row0 + r_in;
            uint4 fv[NPF], fnext[NPF];
            auto fetch_fwd = [&](int c, uint4 (&dst)[NPF]) {
#pragma unroll
                for (int i = 0; i < NPF; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
                if constexpr (DU) {
                    if (!row_ok) return;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int col = ti.n0 + c * 32 + 8 * i;
                        if (col >= p.n_dim) break;
                        if (MODE == BW_DU_RELU) {
                            dst[i] = __ldg(reinterpret_cast<const uint4*>(p.h + r_du * p.n_dim + col));
                        } else {
                            const __nv_bfloat16* pre = p.pre + r_du * (int64_t)(2 * p.n_dim);
                            dst[i] = __ldg(reinterpret_cast<const uint4*>(pre + col));
                            dst[(4 + i) % NPF] = __ldg(reinterpret_cast<const uint4*>(pre + p.n_dim + col));
                        }
                    }
                }
            };
            if (DU) fetch_fwd(0, fnext);
            // dx rows: the destination row (the token, when scattering) before the
            // wait; -1 for rows past the tile.  dx_dst[k4]: the row this lane
            // stores in step k4 of the row-piece path (rows 4 k4 + lane / 8)
            long long dx_row = -1;
            if (MODE == BW_DX && r_in < ti.rows) {
                const int64_t r = (int64_t)ti.row0 + r_in;
                dx_row = p.row_token ? (long long)p.row_token[r] : (long long)r;
            }
            long long dx_dst[8];
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4)
                dx_dst[k4] = MODE == BW_DX ? __shfl_sync(0xffffffffu, dx_row, 4 * k4 + (lane >> 3)) : -1;
            const bool got = wait_bar(smem_u32(&tfull_bar[acc]), acc_par, w);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BW_BN);
            const bool empty_k = MODE == BW_WGT && ti.k_rows == 0;
#pragma unroll 1
            for (int c = 0; c < BW_BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tbase + c * 32, v);
                if (DU) {
#pragma unroll
                    for (int i = 0; i < NPF; ++i) fv[i] = fnext[i];
                    if (c + 1 < BW_BN / 32) fetch_fwd(c + 1, fnext);
                }
                tmem_wait_ld();
                const int col0 = ti.n0 + c * 32;
                if (MODE == BW_WGT) {
                    // the warp's 32 rows x 32 fp32 columns go through a swizzled
                    // staging buffer: one TMA store when all 32 rows are the
                    // expert's, else 128-byte row pieces (8 lanes per row)
                    const uint32_t ebuf = ebuf0 + (nchunk & 1u) * (32 * 128);
                    const uint32_t row_sw = ebuf + lane * 128 + ((lane & 7) << 4);
                    if (lane == 0) bulk_wait_read<1>();   // the store that last read this buffer is done
                    __syncwarp();
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const uint32_t x0 = empty_k ? 0u : v[4 * g], x1 = empty_k ? 0u : v[4 * g + 1];
                        const uint32_t x2 = empty_k ? 0u : v[4 * g + 2], x3 = empty_k ? 0u : v[4 * g + 3];
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_sw ^ (uint32_t)(g << 4)),
                                     "r"(x0), "r"(x1), "r"(x2), "r"(x3)
                                     : "memory");
                    }
                    const int wrow0 = ti.m0 + q * 32;   // the warp's first row
                    if (wrow0 + 32 <= p.m_dim) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) tma_store_2d(&tmOut, ebuf, col0, ti.e * p.m_dim + wrow0);
                    } else {
                        __syncwarp();
                        const int gi = lane & 7;
                        const bool col_ok = col0 + 4 * gi < p.n_dim;
#pragma unroll
                        for (int k4 = 0; k4 < 8; ++k4) {
                            const int r = 4 * k4 + (lane >> 3);
                            uint4 val;
                            const uint32_t srcp = ebuf + r * 128 + ((gi ^ (r & 7)) << 4);
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                         : "r"(srcp)
                                         : "memory");
                            if (wrow0 + r < p.m_dim && col_ok)
                                *reinterpret_cast<uint4*>(p.out + ((int64_t)ti.e * p.m_dim + wrow0 + r) * p.n_dim +
                                                          col0 + 4 * gi) = val;
                        }
                    }
                    if (lane == 0) bulk_commit();
                    __syncwarp();
                    ++nchunk;
                    continue;
                }
                if constexpr (MODE == BW_DX) {
                    // fp32 rows through the staging buffer: one TMA store when the
                    // warp's 32 rows are compact rows of this tile, else 128-byte
                    // row pieces (8 lanes per row) to their token rows
                    const uint32_t ebuf = ebuf0 + (nchunk & 1u) * (32 * 128);
                    const uint32_t row_sw = ebuf + lane * 128 + ((lane & 7) << 4);
                    if (lane == 0) bulk_wait_read<1>();
                    __syncwarp();
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_sw ^ (uint32_t)(g << 4)),
                                     "r"(v[4 * g]), "r"(v[4 * g + 1]), "r"(v[4 * g + 2]), "r"(v[4 * g + 3])
                                     : "memory");
                    if (p.row_token == nullptr && q * 32 + 32 <= ti.rows) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) tma_store_2d(&tmOut, ebuf, col0, ti.row0 + q * 32);
                    } else {
                        __syncwarp();
                        const int gi = lane & 7;
                        const bool col_ok = col0 + 4 * gi < p.n_dim;
#pragma unroll
                        for (int k4 = 0; k4 < 8; ++k4) {
                            const int r = 4 * k4 + (lane >> 3);
                            uint4 val;
                            const uint32_t srcp = ebuf + r * 128 + ((gi ^ (r & 7)) << 4);
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                         : "r"(srcp)
                                         : "memory");
                            if (dx_dst[k4] >= 0 && col_ok)
                                *reinterpret_cast<uint4*>(p.out + (int64_t)dx_dst[k4] * p.n_dim + col0 + 4 * gi) = val;
                        }
                    }
                    if (lane == 0) bulk_commit();
                    __syncwarp();
                    ++nchunk;
                    continue;
                }
                if constexpr (MODE == BW_DU_RELU) {
                    // dU = dA where H > 0: bf16, two 32-column chunks per 128-byte
                    // staging row, then one TMA store per 64 columns (row pieces
                    // when some of the warp's rows are past the tile)
                    const uint32_t half = (uint32_t)(c & 1);
                    const uint32_t ebuf = ebuf0 + (nchunk & 1u) * (32 * 128);
                    const uint32_t row_sw = ebuf + lane * 128 + ((lane & 7) << 4);
                    if (half == 0) {
                        if (lane == 0) bulk_wait_read<1>();
                        __syncwarp();
                    }
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint32_t* hw = reinterpret_cast<const uint32_t*>(&fv[h % NPF]);
                        uint32_t pk[4];
#pragma unroll
                        for (int h2 = 0; h2 < 4; ++h2) {
                            const float a0 = bf16lo(hw[h2]) > 0.f ? __uint_as_float(v[8 * h + 2 * h2]) : 0.f;
                            const float a1 = bf16hi(hw[h2]) > 0.f ? __uint_as_float(v[8 * h + 2 * h2 + 1]) : 0.f;
                            pk[h2] = pack_bf16x2(a0, a1);
                        }
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_sw ^ ((half * 4 + h) << 4)),
                                     "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                                     : "memory");
                    }
                    if (half == 1) {
                        const int pcol0 = col0 - 32;   // first column of the 64-column pair
                        if (q * 32 + 32 <= ti.rows) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) tma_store_2d(&tmOut, ebuf, pcol0, ti.row0 + q * 32);
                        } else {
                            __syncwarp();
                            const int gi = lane & 7;
                            const bool col_ok = pcol0 + 8 * gi < p.n_dim;
#pragma unroll
                            for (int k4 = 0; k4 < 8; ++k4) {
                                const int rr = 4 * k4 + (lane >> 3);
                                uint4 val;
                                const uint32_t srcp = ebuf + rr * 128 + ((gi ^ (rr & 7)) << 4);
                                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                             : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                             : "r"(srcp)
                                             : "memory");
                                if (q * 32 + rr < ti.rows && col_ok)
                                    *reinterpret_cast<uint4*>(p.du + ((int64_t)ti.row0 + q * 32 + rr) * p.n_dim + pcol0 +
                                                              8 * gi) = val;
                            }
                        }
                        if (lane == 0) bulk_commit();
                        __syncwarp();
                        ++nchunk;
                    }
                    continue;
                }
                if (r_in >= ti.rows) continue;
                const int64_t r = (int64_t)ti.row0 + r_in;
                {
                // dU from dA = the accumulator
#pragma unroll
                for (int j0 = 0; j0 < 32; j0 += 8) {
                    const int col = col0 + j0;
                    if (col >= p.n_dim) break;
                    uint32_t pk[4], pk2[4];
                    if (MODE == BW_DU_RELU) {
                        const uint32_t* hw = reinterpret_cast<const uint32_t*>(&fv[(j0 / 8) % NPF]);
#pragma unroll
                        for (int h2 = 0; h2 < 4; ++h2) {
                            const float a0 = bf16lo(hw[h2]) > 0.f ? __uint_as_float(v[j0 + 2 * h2]) : 0.f;
                            const float a1 = bf16hi(hw[h2]) > 0.f ? __uint_as_float(v[j0 + 2 * h2 + 1]) : 0.f;
                            pk[h2] = pack_bf16x2(a0, a1);
                        }
                        *reinterpret_cast<uint4*>(p.du + r * p.n_dim + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    } else {
                        const uint32_t* gw = reinterpret_cast<const uint32_t*>(&fv[(j0 / 8) % NPF]);
                        const uint32_t* uw = reinterpret_cast<const uint32_t*>(&fv[(4 + j0 / 8) % NPF]);
#pragma unroll
                        for (int h2 = 0; h2 < 4; ++h2) {
                            float dgo[2], duo[2];
#pragma unroll
                            for (int z = 0; z < 2; ++z) {
                                const float g = z ? bf16hi(gw[h2]) : bf16lo(gw[h2]);
                                const float up = z ? bf16hi(uw[h2]) : bf16lo(uw[h2]);
                                const float da = __uint_as_float(v[j0 + 2 * h2 + z]);
                                const float sg = sigmoidf_(g);
                                dgo[z] = da * up * (sg * (1.f + g * (1.f - sg)));   // silu'(g) = s (1 + g (1 - s))
                                duo[z] = da * (g * sg);                              // silu(g)
                            }
                            pk[h2] = pack_bf16x2(dgo[0], dgo[1]);
                            pk2[h2] = pack_bf16x2(duo[0], duo[1]);
                        }
                        __nv_bfloat16* o = p.du + r * (int64_t)(2 * p.n_dim);
                        *reinterpret_cast<uint4*>(o + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        *reinterpret_cast<uint4*>(o + p.n_dim + col) = make_uint4(pk2[0], pk2[1], pk2[2], pk2[3]);
                    }
                }
                }
            }
            tc_fence_before();
            mbar_arrive_relaxed(smem_u32(&tempty_bar[acc]));
        }
        if ((MODE == BW_WGT || MODE == BW_DX || MODE == BW_DU_RELU) && lane == 0) bulk_wait_all();   // TMA stores landed
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, BW_TMEM_COLS);
}

// dY[r] = bf16(row_gate[r] * dout[row_token[r]]): one warp per compact row.
__global__ void __launch_bounds__(256)
dy_gather_kernel(const __nv_bfloat16* __restrict__ dout, const int32_t* __restrict__ offsets, int N,
                 const int32_t* __restrict__ row_token, const float* __restrict__ row_gate, int d,
                 __nv_bfloat16* __restrict__ dy) {
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= offsets[N]) return;
    const float g = row_gate[r];
    const __nv_bfloat16* src = dout + (int64_t)row_token[r] * d;
    __nv_bfloat16* dst = dy + r * d;
    for (int c = lane * 8; c < d; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + c);
        const uint32_t* wv = reinterpret_cast<const uint32_t*>(&v);
        uint32_t o[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) o[h] = pack_bf16x2(g * bf16lo(wv[h]), g * bf16hi(wv[h]));
        *reinterpret_cast<uint4*>(dst + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// out[e][c] = sum over expert e's rows of src[r][col_off + c] (fp32, rows in
// order): the bias gradients.  One thread per (expert, column).
__global__ void __launch_bounds__(256)
col_sum_kernel(const __nv_bfloat16* __restrict__ src, int64_t ld, int col_off, int width,
               const int32_t* __restrict__ offsets, int N, float* __restrict__ out) {
    pdl_wait();
    pdl_launch();
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int e = blockIdx.y;
    if (c >= width || e >= N) return;
    float acc = 0.f;
    for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r) acc += __bfloat162float(src[r * ld + col_off + c]);
    out[(int64_t)e * width + c] = acc;
}

// top-2 (or fp32 row output): dx[t] = sum over kept r of dxe[offsets[idx] + pos]
// (fp32, rank order); zero when every assignment of t was dropped.
__global__ void __launch_bounds__(256)
dx_combine_kernel(const float* __restrict__ dxe, const int32_t* __restrict__ idx, const int32_t* __restrict__ pos,
                  const uint8_t* __restrict__ drop, const int32_t* __restrict__ offsets, int64_t T, int d, int k,
                  float* __restrict__ dx) {
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    int64_t row[2] = {-1, -1};
    for (int r = 0; r < k; ++r)
        if (!drop[t * k + r]) row[r] = (int64_t)offsets[idx[t * k + r]] + pos[t * k + r];
    for (int c = lane; c < d; c += 32) {
        float acc = 0.f;
        for (int r = 0; r < k; ++r)
            if (row[r] >= 0) acc += dxe[row[r] * d + c];
        dx[t * d + c] = acc;
    }
}

// rows of dropped tokens (top-1 scatter path): dx[t] = 0
__global__ void __launch_bounds__(256)
dx_zero_dropped_kernel(const uint8_t* __restrict__ drop, int64_t T, int d, float* __restrict__ dx) {
    pdl_wait();
    pdl_launch();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T || !drop[t]) return;
    for (int c = lane; c < d; c += 32) dx[t * d + c] = 0.f;
}

template <int MODE>
cudaError_t run_bwd(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const CUtensorMap& o,
                    const BwdParams& p, cudaStream_t s) {
    int sms = 0;
    cudaError_t err = device_sm_count(&sms);
    if (err != cudaSuccess) return err;
    err = once_per_device(reinterpret_cast<const void*>(bwd_gemm_kernel<MODE>), [](const void* k) {
        return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BW_SMEM);
    });
    if (err != cudaSuccess) return err;
    return launch_k(bwd_gemm_kernel<MODE>, dim3((unsigned)sms), dim3(BW_THREADS), BW_SMEM, s, 1, a, b, b2, o, p);
}

// [rows, n] fp32 (dW as [groups * m, n], or compact dx rows) as an fp32
// epilogue's TMA store target:
// boxes of 32 rows x 32 columns (128 bytes), 128-byte swizzle
bool f32_out_map(CUtensorMap* m, const float* out, int64_t rows, int n) {
    using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn enc = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeFn) nullptr;
        return reinterpret_cast<EncodeFn>(ptr);
    }();
    if (!enc || out == nullptr || n % 4 != 0 || rows < 1) return false;
    cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)n * 4};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(out), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An MN-major operand: the blocked 3-D map (one TMA load of `blocks` 64-column
// blocks per stage) when its shape allows, else the 2-D map (one load per
// block); *blocked says which.
bool mn_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t row_stride, int blocks,
            bool* blocked) {
    *blocked = make_map_bf16_mn_blocks(m, base, rows, cols, row_stride, BW_BK, blocks);
    return *blocked || make_map_bf16_strided(m, base, rows, cols, row_stride, BW_BK);
}

}  // namespace

// Plain tensor-core products of the router backward (router_bwd.cu), over
// groups of rows given by `offsets` [groups + 1] (device):
//   rows: out[r, :] = A[r, :] B with A [rows, K] K-major, B [K, n] read MN-major;
//   weights: out[g] = A_g^T B_g over each group's rows, A [rows, m] and B
//   [rows, n] both read MN-major (out [groups, m, n]).
// Outputs fp32.
cudaError_t launch_tc_rows_f32(const void* A, int64_t rows, int K, const void* B, int n, const int32_t* offsets,
                               float* out, int32_t* status, cudaStream_t s) {
    CUtensorMap ma, mb;
    bool bb = false;
    if (!make_map_bf16(&ma, A, rows, K, BW_BM) || !mn_map(&mb, B, K, n, n, 4, &bb)) return cudaErrorInvalidValue;
    BwdParams p{};
    p.mn3 = bb ? 2 : 0;
    p.offsets = offsets;
    p.N = 1;
    p.n_dim = n;
    p.k_dim = K;
    p.out = out;
    p.status = status;
    p.limit_ns = kWaitLimitNs;
    CUtensorMap mo;
    if (!f32_out_map(&mo, out, rows, n)) return cudaErrorInvalidValue;
    return run_bwd<BW_DX>(ma, mb, mb, mo, p, s);
}

cudaError_t launch_tc_weights_f32(const void* A, int64_t rows, int m, const void* B, int n, const int32_t* offsets,
                                  int groups, float* out, int32_t* status, cudaStream_t s) {
    CUtensorMap ma, mb;
    bool ba = false, bb = false;
    if (!mn_map(&ma, A, rows, m, m, 2, &ba) || !mn_map(&mb, B, rows, n, n, 4, &bb)) return cudaErrorInvalidValue;
    BwdParams p{};
    p.mn3 = (ba ? 1 : 0) | (bb ? 2 : 0);
    p.offsets = offsets;
    p.N = groups;
    p.m_dim = m;
    p.n_dim = n;
    p.out = out;
    p.status = status;
    p.limit_ns = kWaitLimitNs;
    CUtensorMap mo;
    if (!f32_out_map(&mo, out, (int64_t)groups * m, n)) return cudaErrorInvalidValue;
    return run_bwd<BW_WGT>(ma, mb, mb, mo, p, s);
}

cudaError_t launch_expert_backward_tc(const BwdArgs& a, cudaStream_t s) {
    const int64_t R = a.R_cap > 0 ? a.R_cap : 1;
    const bool sw = a.act == MOE_SWIGLU;
    const int d = a.d, dff = a.d_ff, N = a.N;
    cudaError_t err;
    // 1. the forward's first GEMM again: H (and the SwiGLU pre-activations)
    FfnArgs f{};
    f.dtype = MOE_BF16;
    f.act = a.act;
    f.N = N;
    f.d = d;
    f.d_ff = dff;
    f.R_cap = a.R_cap;
    f.xe = a.xe;
    f.offsets = a.offsets;
    f.w1 = a.w1;
    f.b1 = a.b1;
    f.w3 = a.w3;
    f.b3 = a.b3;
    f.h = a.h;
    f.pre_out = sw ? a.pre : nullptr;
    f.stage1_only = true;
    f.hdr = a.hdr;
    if ((err = launch_expert_ffn_tc(f, s)) != cudaSuccess) return err;
    // 2. dY = gate * dout[token]
    const unsigned rows_grid = (unsigned)((R + 7) / 8);
    if ((err = launch_k(dy_gather_kernel, dim3(rows_grid), dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.dout), a.offsets, N, a.row_token, a.row_gate, d,
                        reinterpret_cast<__nv_bfloat16*>(a.dy))) != cudaSuccess)
        return err;
    CUtensorMap m_dy, m_w2, m_du, m_w1, m_w3, m_xe, m_h, m_a2, m_b2;
    // 3. dA = dY W2 -> dU (dG | dUp)
    bool bw2 = false;
    if (!make_map_bf16(&m_dy, a.dy, R, d, BW_BM) || !mn_map(&m_w2, a.w2, (int64_t)N * d, dff, dff, 4, &bw2))
        return cudaErrorInvalidValue;
    BwdParams p{};
    p.mn3 = bw2 ? 2 : 0;
    p.offsets = a.offsets;
    p.N = N;
    p.status = &a.hdr->status;
    p.limit_ns = kWaitLimitNs;
    p.n_dim = dff;
    p.k_dim = d;
    p.h = reinterpret_cast<const __nv_bfloat16*>(a.h);
    p.pre = reinterpret_cast<const __nv_bfloat16*>(a.pre);
    p.du = reinterpret_cast<__nv_bfloat16*>(a.du);
    CUtensorMap m_duo;   // ReLU dU [R, d_ff]: the TMA store target, 64 columns x 32 rows
    if (!sw && !make_map_bf16(&m_duo, a.du, R, dff, 32)) return cudaErrorInvalidValue;
    err = sw ? run_bwd<BW_DU_SWIGLU>(m_dy, m_w2, m_w2, m_dy, p, s)
             : run_bwd<BW_DU_RELU>(m_dy, m_w2, m_w2, m_duo, p, s);
    if (err != cudaSuccess) return err;
    // 4. dx rows = dU W1 (+ dUp W3): K = d_ff (2 d_ff for SwiGLU, W3 for the second half)
    const int kdu = sw ? 2 * dff : dff;
    bool bw1 = false, bw3 = false;
    if (!make_map_bf16(&m_du, a.du, R, kdu, BW_BM) || !mn_map(&m_w1, a.w1, (int64_t)N * dff, d, d, 4, &bw1))
        return cudaErrorInvalidValue;
    if (sw && !mn_map(&m_w3, a.w3, (int64_t)N * dff, d, d, 4, &bw3)) return cudaErrorInvalidValue;
    if (sw && bw1 != bw3) {   // both B tensors of one launch in the same form
        bw1 = bw3 = false;
        if (!make_map_bf16_mn(&m_w1, a.w1, (int64_t)N * dff, d, BW_BK) ||
            !make_map_bf16_mn(&m_w3, a.w3, (int64_t)N * dff, d, BW_BK))
            return cudaErrorInvalidValue;
    }
    BwdParams px = p;
    px.mn3 = bw1 ? 2 : 0;
    px.n_dim = d;
    px.k_dim = kdu;
    px.k_split = sw ? dff : 0;
    px.out = a.top1_scatter ? a.dx : a.dxe;
    px.row_token = a.top1_scatter ? a.row_token : nullptr;
    CUtensorMap m_dxo = m_du;   // compact dx rows (top-2): the TMA store target
    if (!a.top1_scatter && !f32_out_map(&m_dxo, a.dxe, R, d)) return cudaErrorInvalidValue;
    if ((err = run_bwd<BW_DX>(m_du, m_w1, sw ? m_w3 : m_w1, m_dxo, px, s)) != cudaSuccess) return err;
    if (a.top1_scatter) {
        if (a.T > 0 && (err = launch_k(dx_zero_dropped_kernel, dim3((unsigned)((a.T + 7) / 8)), dim3(256), 0, s, 1,
                                       a.drop, a.T, d, a.dx)) != cudaSuccess)
            return err;
    } else if (a.T > 0) {
        if ((err = launch_k(dx_combine_kernel, dim3((unsigned)((a.T + 7) / 8)), dim3(256), 0, s, 1,
                            static_cast<const float*>(a.dxe), a.idx, a.pos, a.drop, a.offsets, a.T, d, a.k,
                            a.dx)) != cudaSuccess)
            return err;
    }
    // 5. weight gradients: dW1 = dU^T X (dW3 = dUp^T X), dW2 = dY^T A
    bool bxe = false, bh = false, ba2 = false;
    if (!mn_map(&m_xe, a.xe, R, d, d, 4, &bxe) || !mn_map(&m_h, a.h, R, dff, dff, 4, &bh))
        return cudaErrorInvalidValue;
    BwdParams pw = p;
    pw.m_dim = dff;
    pw.n_dim = d;
    // dU (dG): the first d_ff columns of each row of the du tensor (row stride kdu)
    if (!mn_map(&m_a2, a.du, R, dff, kdu, 2, &ba2)) return cudaErrorInvalidValue;
    pw.out = a.dw1;
    pw.mn3 = (ba2 ? 1 : 0) | (bxe ? 2 : 0);
    CUtensorMap m_o;
    if (a.dw1) {
        if (!f32_out_map(&m_o, a.dw1, (int64_t)N * dff, d)) return cudaErrorInvalidValue;
        if ((err = run_bwd<BW_WGT>(m_a2, m_xe, m_xe, m_o, pw, s)) != cudaSuccess) return err;
    }
    if (sw && a.dw3) {   // dUp: columns [d_ff, 2 d_ff)
        bool bb2 = false;
        if (!mn_map(&m_b2, reinterpret_cast<const __nv_bfloat16*>(a.du) + dff, R, dff, kdu, 2, &bb2))
            return cudaErrorInvalidValue;
        pw.out = a.dw3;
        pw.mn3 = (bb2 ? 1 : 0) | (bxe ? 2 : 0);
        if (!f32_out_map(&m_o, a.dw3, (int64_t)N * dff, d)) return cudaErrorInvalidValue;
        if ((err = run_bwd<BW_WGT>(m_b2, m_xe, m_xe, m_o, pw, s)) != cudaSuccess) return err;
    }
    if (a.dw2) {
        CUtensorMap m_dy_mn;
        bool bdy = false;
        if (!mn_map(&m_dy_mn, a.dy, R, d, d, 2, &bdy)) return cudaErrorInvalidValue;
        BwdParams p2 = p;
        p2.m_dim = d;
        p2.n_dim = dff;
        p2.out = a.dw2;
        p2.mn3 = (bdy ? 1 : 0) | (bh ? 2 : 0);
        if (!f32_out_map(&m_o, a.dw2, (int64_t)N * d, dff)) return cudaErrorInvalidValue;
        if ((err = run_bwd<BW_WGT>(m_dy_mn, m_h, m_h, m_o, p2, s)) != cudaSuccess) return err;
    }
    // 6. bias gradients
    const dim3 cs_block(256);
    if (a.db1 && (err = launch_k(col_sum_kernel, dim3((unsigned)((dff + 255) / 256), (unsigned)N), cs_block, 0, s, 1,
                                 static_cast<const __nv_bfloat16*>(a.du), (int64_t)kdu, 0, dff, a.offsets, N,
                                 a.db1)) != cudaSuccess)
        return err;
    if (sw && a.db3 && (err = launch_k(col_sum_kernel, dim3((unsigned)((dff + 255) / 256), (unsigned)N), cs_block, 0, s,
                                       1, static_cast<const __nv_bfloat16*>(a.du), (int64_t)kdu, dff, dff, a.offsets,
                                       N, a.db3)) != cudaSuccess)
        return err;
    if (a.db2 && (err = launch_k(col_sum_kernel, dim3((unsigned)((d + 255) / 256), (unsigned)N), cs_block, 0, s, 1,
                                 static_cast<const __nv_bfloat16*>(a.dy), (int64_t)d, 0, d, a.offsets, N, a.db2)) !=
                     cudaSuccess)
        return err;
    return cudaSuccess;
}

}  // namespace moe
