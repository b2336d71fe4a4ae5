// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every expert e and every compact row of e (rows
// [offsets[e], offsets[e+1]) of A):
//   stage 1, ReLU   : H = relu(A W1[e]^T + b1[e])
//   stage 1, SwiGLU : H = silu(A W1[e]^T + b1[e]) * (A W3[e]^T + b3[e])
//   stage 2         : Y = H W2[e]^T + b2[e]            (compact rows), or
//   stage 2, scatter: out[row_token[r]] = row_gate[r] * (H W2[e]^T + b2[e])[r]
//                     (expert parallelism: out is that of GPU row_rank[r], reached
//                     through a peer pointer; row_gate may be absent)
// which is the expert FFN of "From Switch Transformer to GLaM" (FFN(x) =
// W2 s(W1 x)), the Mixtral SwiGLU expert of CMU 10-423 Lecture 16 section 2.3,
// and the gate-scaled top-1 combine y = p_{i*} E_{i*}(x) of the GLaM page.
//
// Kernel design (persistent, one CTA per SM, 192 threads, warp-specialised):
//   warp 0   TMA producer: per stage two 64-deep K boxes (128-byte swizzle) of
//            A (128 rows) and of B into an mbarrier ring.
//   warp 1   TMEM allocator + MMA issuer: tcgen05.mma kind::f16, bf16 x bf16 ->
//            fp32 in TMEM, N = 256; two 256-column accumulators (all 512
//            columns) so the epilogue of tile i overlaps the main loop of i+1.
//   warps 2-5 epilogue: tcgen05.ld 32x32b (thread = row), bias, activation,
//            gate, bf16 pack, 16-byte stores (optionally scattered to token rows).
// Two variants share this code:
//   single   one CTA owns a 128 x 256 tile (M=128 MMA); a stage is 32 KB of A
//            plus 64 KB of B (128 deep in K), 2 stages.
//   pair     a cluster of two CTAs owns a 256 x 256 tile with cta_group::2
//            MMAs (M=256) issued by the pair's leader: each CTA loads its own
//            128 rows of A and its own 128 rows of B, so a stage is 64 KB per CTA
//            (128 deep in K) and 3 stages fit -- half the shared-memory traffic
//            per MMA.  Both CTAs' loads complete on the leader's full
//            barrier (only the leader expects the bytes), the leader's MMA
//            commits release both CTAs' stages and accumulators, and both CTAs'
//            epilogues release the leader's accumulator.
// SwiGLU: the 256 B rows of a tile are 128 rows of W1 and the same 128 rows of
// W3 (single: stacked in one stage; pair: W1 in the leader, W3 in the peer), so
// one N=256 MMA produces the gate and up halves side by side in TMEM.
// Tiles: an expert's rows are cut into m-tiles; the tile list is expert-major
// with m-tiles grouped by 8 inside an expert (concurrent CTAs share B columns and
// A rows in L2), n-tiles fastest when there are at most 4 of them.  Rows past
// an expert's end inside its last m-tile belong to the next expert (or are
// zero-filled out of bounds); the MMA computes them and the epilogue masks them.
// Every wait on an mbarrier is bounded: on expiry the kernel latches
// MOE_ERR_TIMEOUT, stops issuing work, waits (bounded) for its own copies and
// MMAs in flight, frees TMEM and returns.
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "tc_common.cuh"

namespace moe {
using namespace tc;
namespace {

constexpr int BM = 128;          // rows per CTA
constexpr int BN = 256;          // MMA N (and TMEM columns per accumulator)
constexpr int BK = 64;           // 64 bf16 = one 128-byte swizzle row (one TMA box wide)
constexpr int KSUB = 2;          // K boxes per pipeline stage: 128-deep stages, 8 MMAs per barrier round trip
constexpr int BKS = BK * KSUB;   // K per stage
constexpr int A_SUB = BM * BK * 2;   // one A box (16 KB)
constexpr int A_BYTES = A_SUB * KSUB;
constexpr int TMEM_COLS = 512;
constexpr int GEMM_THREADS = 192;
constexpr int GROUP_M = 8;

template <bool PAIR>
struct GemmShape {
    static constexpr int TILE_M = PAIR ? 2 * BM : BM;             // rows per tile
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;             // B rows loaded per CTA
    static constexpr int B_SUB = B_ROWS * BK * 2;                 // one K box of B rows
    static constexpr int B_BYTES = B_SUB * KSUB;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // 128-deep stages measured faster than 64-deep ones at the same bytes in
    // flight (Switch-Base 599 -> 586 us, top-2 940 -> 900 us, Mixtral 9.8 -> 9.0 ms)
    static constexpr int STAGES = PAIR ? 3 : 2;
    static constexpr int EPI_BYTES = 2 * 4 * 32 * 128;            // per epilogue warp: 2 x (32 rows x 128 B)
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024;
    static_assert((STAGES * STAGE_BYTES) % 1024 == 0, "epilogue staging buffers start 1024-byte aligned");
    static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, BN);
};

enum { EPI_RELU = 0, EPI_SWIGLU = 1, EPI_BIAS = 2, EPI_SCATTER = 3 };

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
    const float* row_gate;        // scatter: nullable (no gate)
    void* const* out_ptrs;        // scatter to several GPUs: row r goes to out_ptrs[row_rank[r]]
    const int32_t* row_rank;
    __nv_bfloat16* pre_out;       // SwiGLU (optional): the pre-activations W1 x + b1 | W3 x + b3, [R, 2 n_dim]
    // 1: tiles in reverse order.  The second GEMM starts with the last experts,
    // whose rows of H the first GEMM wrote last and L2 still holds.
    int reverse;
    int32_t* status;
    long long limit_ns;
};

struct TileInfo {
    int e, row0, rows, n0;
};

// tile -> (expert, first compact row, valid rows, first output column)
template <int TILE_M>
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
    const int mt = (rows_e + TILE_M - 1) / TILE_M;
    const int local = tile - prefix[e];
    const int per_group = GROUP_M * ntn;
    const int g = local / per_group;
    const int first_m = g * GROUP_M;
    const int gsz = min(mt - first_m, GROUP_M);
    const int rem = local - g * per_group;
    // few n-tiles (a second GEMM with d <= 1024): n fastest, so the tiles that
    // share one block of A rows run at the same time and it is read from DRAM
    // once (Switch-Base stage 2: 764 -> 750 MB read, top-2: 956 -> 879 MB);
    // otherwise m fastest in groups of GROUP_M (tiles sharing B columns)
    const int m_blk = ntn <= 4 ? first_m + rem / ntn : first_m + rem % gsz;
    const int n_blk = ntn <= 4 ? rem % ntn : rem / gsz;
    TileInfo ti;
    ti.e = e;
    ti.row0 = off[e] + m_blk * TILE_M;
    ti.rows = min(TILE_M, rows_e - m_blk * TILE_M);
    ti.n0 = n_blk * bn_out;
    return ti;
}

// z sigmoid(z) = z / (1 + e^-z); e^-z = 2^(-z log2 e) -> inf for very negative
// z, where the fast division gives the limit 0
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.f + fast_exp2(-z * kLog2e)); }

template <int EPI, bool PAIR>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmOut,
                    const GemmParams p) {
    using S = GemmShape<PAIR>;
    constexpr int BN_OUT = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[S::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[S::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_off[129];
    __shared__ int s_prefix[129];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0 = the pair's leader
    const bool leader = rank == 0;
    const int first_tile = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
    const int tile_step = PAIR ? (int)ncluster_x() : (int)gridDim.x;
    const int N = p.N;
    if (tid == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull_bar[a]), 1);
            mbar_init(smem_u32(&tempty_bar[a]), PAIR ? 256 : 128);
        }
        mbar_init(smem_u32(&done_bar), 1);
        s_abort = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        if (PAIR) tmem_alloc_pair(&s_tmem, TMEM_COLS);
        else tmem_alloc(&s_tmem, TMEM_COLS);
    }
    pdl_wait();   // the compact rows and offsets are ready from here on
    pdl_launch();
    for (int i = tid; i <= N; i += GEMM_THREADS) s_off[i] = p.offsets[i];
    __syncthreads();
    const int ntn = (p.n_dim + BN_OUT - 1) / BN_OUT;
    if (warp == 2) {
        // tiles per expert and their exclusive prefix (one warp, N <= 128: four
        // experts per lane, then a shuffle scan over the lanes)
        int cnt[4], sum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = lane * 4 + j;
            cnt[j] = e < N ? ((s_off[e + 1] - s_off[e] + S::TILE_M - 1) / S::TILE_M) * ntn : 0;
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
        if (lane == 31) s_prefix[N] = incl;   // all tiles
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();   // the peer's barriers exist before any cross-CTA signal
    tc_fence_after();

    const uint32_t tmem_base = s_tmem;
    const int total = s_prefix[N];
    const int nkb = (p.k_dim + BKS - 1) / BKS;   // stages per tile (the last box of the last one may be K padding)
    const Waiter w{&s_abort, p.status, p.limit_ns};

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            // With few n-tiles (n fastest), an expert's weight columns are read by
            // each of its m-blocks, and the m-blocks of an expert at a wave's end
            // run a wave later: the B lines are loaded evict-last, so the stream
            // of A rows (read by an m-block's n-tiles at about the same time, then
            // dead) does not evict weights that are read again.  Stage-2 DRAM
            // reads over the compulsory H + W2 (ncu, several captures):
            // Switch-Base 1.052x -> 1.03-1.04x, top-2 1.083x -> 1.04-1.05x (A
            // evict-first as well: 1.29x, the n-tiles then miss each other's rows).
            const bool hint = ntn <= 4;
            const uint64_t pol_b = l2_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            int last_par[S::STAGES];
#pragma unroll
            for (int s = 0; s < S::STAGES; ++s) last_par[s] = -1;
            bool ok = true;
            for (int tile = first_tile; tile < total && ok; tile += tile_step) {
                const TileInfo ti = decode_tile<S::TILE_M>(p.reverse ? total - 1 - tile : tile, s_prefix, s_off, N, ntn, BN_OUT);
                const int arow = ti.row0 + (int)rank * BM;
                const int brow = ti.e * p.n_dim + ti.n0 + ((PAIR && EPI != EPI_SWIGLU) ? (int)rank * (BN / 2) : 0);
                const CUtensorMap* bmap = (EPI == EPI_SWIGLU && PAIR && rank == 1) ? &tmB3 : &tmB;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(smem_u32(&empty_bar[stage]), phase ^ 1u, w)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t a_dst = smem_u32(smem + stage * S::STAGE_BYTES);
                    const uint32_t b_dst = a_dst + A_BYTES;
                    if (PAIR) {
                        const uint32_t fb_leader = map_to_rank(fb, 0);
                        if (leader) mbar_expect_tx(fb, 2 * S::STAGE_BYTES);   // both CTAs' bytes
#pragma unroll
                        for (int j = 0; j < KSUB; ++j) {
                            tma_load_2d_pair(a_dst + j * A_SUB, &tmA, fb_leader, kb * BKS + j * BK, arow);
                            if (hint)
                                tma_load_2d_pair_hint(b_dst + j * S::B_SUB, bmap, fb_leader, kb * BKS + j * BK, brow, pol_b);
                            else
                                tma_load_2d_pair(b_dst + j * S::B_SUB, bmap, fb_leader, kb * BKS + j * BK, brow);
                        }
                    } else {
                        mbar_expect_tx(fb, S::STAGE_BYTES);
#pragma unroll
                        for (int j = 0; j < KSUB; ++j) {
                            const int k0 = kb * BKS + j * BK;
                            tma_load_2d(a_dst + j * A_SUB, &tmA, fb, k0, arow);
                            if (EPI == EPI_SWIGLU) {   // W1 rows, then the same W3 rows
                                tma_load_2d(b_dst + j * S::B_SUB, &tmB, fb, k0, brow);
                                tma_load_2d(b_dst + j * S::B_SUB + S::B_SUB / 2, &tmB3, fb, k0, brow);
                            } else if (hint) {
                                tma_load_2d_hint(b_dst + j * S::B_SUB, &tmB, fb, k0, brow, pol_b);
                            } else {
                                tma_load_2d(b_dst + j * S::B_SUB, &tmB, fb, k0, brow);
                            }
                        }
                    }
                    last_par[stage] = (int)phase;
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every load this thread issued has landed before the CTA retires:
            // single -- its full barrier completed; pair -- the leader's MMA released
            // the stage (which it does only after the stage's bytes arrived)
            for (int s = 0; s < S::STAGES; ++s) {
                if (last_par[s] < 0) continue;
                if (PAIR) drain_bar(smem_u32(&empty_bar[s]), (uint32_t)last_par[s], p.limit_ns, p.status);
                else drain_bar(smem_u32(&full_bar[s]), (uint32_t)last_par[s], p.limit_ns, p.status);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (the leader, for a pair) ----------------
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true, issued = false;
            for (int tile = first_tile; tile < total && ok; tile += tile_step, ++it) {
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
                    const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
                    // the descriptors' address field counts 16-byte units: the next
                    // 16-wide K slice (32 bytes) of the swizzled rows is +2, the
                    // stage's second K box A_SUB (B_SUB) bytes on
                    const uint64_t a_desc = umma_desc(a_addr), b_desc = umma_desc(a_addr + A_BYTES);
#pragma unroll
                    for (int j = 0; j < KSUB; ++j) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t ad = a_desc + (uint64_t)((j * A_SUB) >> 4) + 2 * kk;
                            const uint64_t bd = b_desc + (uint64_t)((j * S::B_SUB) >> 4) + 2 * kk;
                            const uint32_t accf = (kb | j | kk) != 0 ? 1u : 0u;
                            if (PAIR) umma_f16_pair(d_tmem, ad, bd, S::IDESC, accf);
                            else umma_f16(d_tmem, ad, bd, S::IDESC, accf);
                        }
                    }
                    // frees the stage (in both CTAs of a pair) when these MMAs finish
                    if (PAIR) umma_commit_pair(smem_u32(&empty_bar[stage]), 0x3);
                    else umma_commit(smem_u32(&empty_bar[stage]));
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) {
                    if (PAIR) umma_commit_pair(smem_u32(&tfull_bar[acc]), 0x3);
                    else umma_commit(smem_u32(&tfull_bar[acc]));
                }
            }
            // all MMAs issued by this thread have completed before TMEM is freed
            if (issued) {
                if (PAIR) umma_commit_pair(smem_u32(&done_bar), 0x3);
                else umma_commit(smem_u32(&done_bar));
                drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
            }
        } else if (PAIR && lane == 0 && !leader && first_tile < total) {
            // the peer's TMEM and shared memory are in use until the leader's MMAs end
            drain_bar(smem_u32(&done_bar), 0u, p.limit_ns, p.status);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        // A thread owns one accumulator row.  Per chunk of 64 output columns it
        // reads its row from TMEM, applies bias / activation / gate, packs bf16 and
        // writes the 128-byte row piece to this warp's staging buffer (16-byte
        // granules XOR-swizzled by row, so the writes are bank-conflict free);
        // the warp then stores 4 full rows per instruction (8 lanes x 16 B per
        // row), so every global store instruction writes whole 128-byte lines.
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int r_in_tile = (int)rank * BM + q * 32 + lane;
        // two staging buffers per warp (32 rows x 128 B each, 128-byte swizzled):
        // compact outputs leave them through TMA stores issued by lane 0
        const uint32_t ebuf0 = smem_u32(smem + S::STAGES * S::STAGE_BYTES + q * 2 * 32 * 128);
        constexpr bool TMA_OUT = EPI != EPI_SCATTER;
        uint32_t nchunk = 0;   // chunks staged so far (buffer = nchunk & 1; one bulk group each)
        const uint32_t tempty_leader0 = PAIR ? map_to_rank(smem_u32(&tempty_bar[0]), 0) : 0u;
        const uint32_t tempty_leader1 = PAIR ? map_to_rank(smem_u32(&tempty_bar[1]), 0) : 0u;
        constexpr int CW = 64;                  // output columns per chunk
        int it = 0;
        for (int tile = first_tile; tile < total; tile += tile_step, ++it) {
            const TileInfo ti = decode_tile<S::TILE_M>(p.reverse ? total - 1 - tile : tile, s_prefix, s_off, N, ntn, BN_OUT);
            const int acc = it & 1;
            const uint32_t acc_par = (uint32_t)((it >> 1) & 1);
            // the row's destination (and, scattering, its token and gate) are
            // fetched before the accumulator is waited for
            const bool valid = r_in_tile < ti.rows;
            const int64_t grow = (int64_t)ti.row0 + r_in_tile;
            int64_t orow = grow;
            float g = 1.f;
            __nv_bfloat16* obase = p.out;   // this row's destination tensor
            if (EPI == EPI_SCATTER && valid) {
                orow = p.row_token[grow];
                if (p.row_gate) g = p.row_gate[grow];
                if (p.row_rank) obase = reinterpret_cast<__nv_bfloat16*>(p.out_ptrs[p.row_rank[grow]]);
            }
            __nv_bfloat16* my_dst = valid ? obase + orow * (int64_t)p.out_ld : nullptr;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const __nv_bfloat16* bias_e = p.bias ? p.bias + (int64_t)ti.e * p.n_dim : nullptr;
            const __nv_bfloat16* bias3_e = p.bias3 ? p.bias3 + (int64_t)ti.e * p.n_dim : nullptr;
            // destination row pointer of the row this lane stores in step k4 (rows
            // 4*k4 + lane/8 of the warp), or null when that row is not valid
            __nv_bfloat16* dst_row[8];
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
                const int r = 4 * k4 + (lane >> 3);
                dst_row[k4] = reinterpret_cast<__nv_bfloat16*>(
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_dst), r));
            }
            const bool got = wait_bar(smem_u32(&tfull_bar[acc]), acc_par, w);
            if (!__all_sync(0xffffffffu, got)) break;   // warp-uniform exit on abort
            tc_fence_after();

            // one chunk of CW output columns from the accumulator values u (and v):
            // bias / activation / gate, bf16 pack, staged rows, 128-byte row stores.
            // hb: whether a bias is added -- a compile-time switch, since the
            // epilogue's instruction count slows the MMA issue on the SM
            // sub-partition it shares with the MMA warp (an always-zero bias add
            // cost 5% of the K = 768 GEMM)
            const bool has_bias = bias_e != nullptr || (EPI == EPI_SWIGLU && bias3_e != nullptr);
            auto emit = [&](auto hb, int c, const uint32_t (&u)[CW],
                            const uint32_t (&v)[EPI == EPI_SWIGLU ? CW : 1]) {
                constexpr bool HB = decltype(hb)::value;
                const int col0 = ti.n0 + c * CW;
                const uint32_t ebuf = ebuf0 + (nchunk & 1u) * (32 * 128);
                // this lane's staged row with its swizzle key in bits 4-6 (ebuf is
                // 1024-byte aligned): granule gi lands at row_sw ^ (gi << 4)
                const uint32_t row_sw = ebuf + lane * 128 + ((lane & 7) << 4);
                if (TMA_OUT) {   // the store that last read this buffer (two chunks ago) is done with it
                    if (lane == 0) bulk_wait_read<1>();
                    __syncwarp();
                }
#pragma unroll
                for (int gi = 0; gi < CW / 8; ++gi) {   // one 16-byte granule = 8 columns
                    const int col = col0 + 8 * gi;
                    float bu[8], bv[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        bu[jj] = 0.f;
                        bv[jj] = 0.f;
                    }
                    if (HB && bias_e && col < p.n_dim) {
                        uint4 bw = __ldg(reinterpret_cast<const uint4*>(bias_e + col));
                        const uint32_t* bp = reinterpret_cast<const uint32_t*>(&bw);
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            bu[2 * h] = bf16lo(bp[h]);
                            bu[2 * h + 1] = bf16hi(bp[h]);
                        }
                    }
                    if (HB && EPI == EPI_SWIGLU && bias3_e && col < p.n_dim) {
                        uint4 bw = __ldg(reinterpret_cast<const uint4*>(bias3_e + col));
                        const uint32_t* bp = reinterpret_cast<const uint32_t*>(&bw);
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            bv[2 * h] = bf16lo(bp[h]);
                            bv[2 * h + 1] = bf16hi(bp[h]);
                        }
                    }
                    uint32_t pk[4];
                    uint32_t pre_g[4], pre_u[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int jj = 8 * gi + 2 * h;
                        float a0 = __uint_as_float(u[jj]);
                        float a1 = __uint_as_float(u[jj + 1]);
                        float v0 = EPI == EPI_SWIGLU ? __uint_as_float(v[EPI == EPI_SWIGLU ? jj : 0]) : 0.f;
                        float v1 = EPI == EPI_SWIGLU ? __uint_as_float(v[EPI == EPI_SWIGLU ? jj + 1 : 0]) : 0.f;
                        if (HB) {
                            a0 += bu[2 * h];
                            a1 += bu[2 * h + 1];
                            v0 += bv[2 * h];
                            v1 += bv[2 * h + 1];
                        }
                        if (EPI == EPI_SWIGLU) {
                            pre_g[h] = pack_bf16x2(a0, a1);
                            pre_u[h] = pack_bf16x2(v0, v1);
                        }
                        if (EPI == EPI_RELU) {
                            pk[h] = pack_relu_bf16x2(a0, a1);
                            continue;
                        } else if (EPI == EPI_SWIGLU) {
                            a0 = silu(a0) * v0;
                            a1 = silu(a1) * v1;
                        } else if (EPI == EPI_SCATTER) {
                            a0 *= g;
                            a1 *= g;
                        }
                        pk[h] = pack_bf16x2(a0, a1);
                    }
                    if (EPI == EPI_SWIGLU && p.pre_out != nullptr && valid && col < p.n_dim) {
                        __nv_bfloat16* pr = p.pre_out + grow * (int64_t)(2 * p.n_dim) + col;
                        *reinterpret_cast<uint4*>(pr) = make_uint4(pre_g[0], pre_g[1], pre_g[2], pre_g[3]);
                        *reinterpret_cast<uint4*>(pr + p.n_dim) = make_uint4(pre_u[0], pre_u[1], pre_u[2], pre_u[3]);
                    }
                    const uint32_t dst = row_sw ^ (uint32_t)(gi << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                                 "r"(pk[2]), "r"(pk[3])
                                 : "memory");
                }
                // all 32 rows of the warp's box belong to this tile: one TMA store
                // (columns past n_dim are clipped by the tensor map); otherwise the
                // rows are stored by the lanes, skipping the rows past the tile
                const bool whole = TMA_OUT && (int)rank * BM + q * 32 + 32 <= ti.rows;
                if (whole) {
                    fence_proxy_async_smem();   // the staged rows are visible to the TMA unit
                    __syncwarp();
                    if (lane == 0) tma_store_2d(&tmOut, ebuf, col0, (int)(ti.row0 + (int)rank * BM + q * 32));
                } else {
                    __syncwarp();
                    const int gi = lane & 7;
                    const bool col_ok = col0 + 8 * gi < p.n_dim;
#pragma unroll
                    for (int k4 = 0; k4 < 8; ++k4) {   // rows 4*k4 .. 4*k4+3 of the warp
                        const int r = 4 * k4 + (lane >> 3);
                        uint4 val;
                        const uint32_t srcp = ebuf + r * 128 + ((gi ^ (r & 7)) << 4);
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                     : "r"(srcp)
                                     : "memory");
                        if (dst_row[k4] != nullptr && col_ok)
                            *reinterpret_cast<uint4*>(dst_row[k4] + col0 + 8 * gi) = val;
                    }
                }
                if (TMA_OUT && lane == 0) bulk_commit();   // one group per chunk, possibly empty
                __syncwarp();
                ++nchunk;
            };
            auto release = [&]() {   // every TMEM read of this accumulator has completed
                tc_fence_before();
                if (PAIR) mbar_arrive_cluster_relaxed(acc ? tempty_leader1 : tempty_leader0);
                else mbar_arrive_relaxed(smem_u32(&tempty_bar[acc]));
            };
            if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll 1
                for (int c = 0; c < BN_OUT / CW; ++c) {
                    uint32_t u[CW], v[CW];
                    tmem_ld32(tbase + c * CW, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
                    tmem_ld32(tbase + c * CW + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
                    tmem_ld32(tbase + BN_OUT + c * CW, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                    tmem_ld32(tbase + BN_OUT + c * CW + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                    tmem_wait_ld();
                    if (c == BN_OUT / CW - 1) release();
                    if (has_bias) emit(std::true_type{}, c, u, v);
                    else emit(std::false_type{}, c, u, v);
                }
            } else {
                // the next chunk's TMEM load is in flight while this chunk is
                // processed; the accumulator is released right after its last load
                constexpr int NC = BN_OUT / CW;
                uint32_t ua[CW], ub[CW], none[1];
                tmem_ld32(tbase, *reinterpret_cast<uint32_t(*)[32]>(&ua[0]));
                tmem_ld32(tbase + 32, *reinterpret_cast<uint32_t(*)[32]>(&ua[32]));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    uint32_t(&cur)[CW] = (c & 1) ? ub : ua;
                    uint32_t(&nxt)[CW] = (c & 1) ? ua : ub;
                    if (c + 1 < NC) {
                        tmem_ld32(tbase + (c + 1) * CW, *reinterpret_cast<uint32_t(*)[32]>(&nxt[0]));
                        tmem_ld32(tbase + (c + 1) * CW + 32, *reinterpret_cast<uint32_t(*)[32]>(&nxt[32]));
                    } else {
                        release();
                    }
                    if (has_bias) emit(std::true_type{}, c, cur, none);
                    else emit(std::false_type{}, c, cur, none);
                    if (c + 1 < NC) tmem_wait_ld();
                }
            }
        }
    }

    if (warp >= 2 && lane == 0 && EPI != EPI_SCATTER) bulk_wait_all();   // this warp's TMA stores have landed
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();   // no CTA leaves while its peer may still signal it
    tc_fence_after();
    if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host ----

struct DeviceInfo {
    int sms = 0;
    bool attr_set[2][4] = {};
};
std::mutex g_mu;
DeviceInfo g_dev[64];

template <int EPI, bool PAIR>
cudaError_t run_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b3, const CUtensorMap& o,
                     const GemmParams& p, cudaStream_t s) {
    using S = GemmShape<PAIR>;
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
        if (!di.attr_set[PAIR][EPI]) {
            err = cudaFuncSetAttribute(grouped_gemm_kernel<EPI, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       S::SMEM_BYTES);
            if (err != cudaSuccess) return err;
            di.attr_set[PAIR][EPI] = true;
        }
        sms = di.sms;
    }
    if constexpr (!PAIR)
        return launch_k(grouped_gemm_kernel<EPI, false>, dim3((unsigned)sms), dim3(GEMM_THREADS), S::SMEM_BYTES, s,
                        1, a, b, b3, o, p);
    else
        return launch_k(grouped_gemm_kernel<EPI, true>, dim3((unsigned)(sms / 2) * 2), dim3(GEMM_THREADS),
                        S::SMEM_BYTES, s, 2, a, b, b3, o, p);
}

// Variant choice: the CTA-pair kernel unless MOE_B200_GEMM=single (kept for
// side-by-side measurement; both compute the same tiles).
bool use_pair() {
    static const bool pair = [] {
        const char* v = getenv("MOE_B200_GEMM");
        return !(v && strcmp(v, "single") == 0);
    }();
    return pair;
}

template <int EPI>
cudaError_t run_gemm_any(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b3, const CUtensorMap& o,
                         const GemmParams& p, cudaStream_t s) {
    return use_pair() ? run_gemm<EPI, true>(a, b, b3, o, p, s) : run_gemm<EPI, false>(a, b, b3, o, p, s);
}

}  // namespace

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

namespace {
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

}  // namespace

// 2-D bf16 tensor [rows, k] (k contiguous), box = box_rows x 64, 128-byte swizzle.
bool tc::make_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int64_t k, int box_rows) {
    return make_map_bf16_strided(map, base, rows, k, k, box_rows);
}

// The first `cols` columns of rows `row_stride` elements apart.
bool tc::make_map_bf16_strided(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t row_stride,
                               int box_rows) {
    EncodeFn enc = get_encode();
    if (!enc) return false;
    const int64_t k = cols;
    cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows, cols] (cols contiguous) as an MN-major operand:
// box = 64 cols x box_rows rows, 128-byte swizzle.
bool tc::make_map_bf16_mn(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
    return make_map_bf16(map, base, rows, cols, box_rows);   // the same box shape: 64 inner elements x rows
}

bool tc::make_map_bf16_mn_blocks(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t row_stride,
                                 int box_rows, int blocks) {
    if (cols % 64 != 0 || row_stride < cols || blocks < 1 || blocks > 8) return false;
    EncodeFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, 128u};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, (cuuint32_t)blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Stage 1 + stage 2 of the bf16 expert FFN on the tensor cores, both
// on CTA pairs unless MOE_B200_GEMM=single.
cudaError_t launch_expert_ffn_tc(const FfnArgs& a, cudaStream_t s) {
    const int64_t R = a.R_cap > 0 ? a.R_cap : 1;
    const bool pair = use_pair();
    const bool swiglu = a.act == MOE_SWIGLU;
    // B rows per CTA and load: pair -> 128; single -> 256 (ReLU) or 128 + 128 (SwiGLU)
    const int b1_box = (swiglu || pair) ? BN / 2 : BN;
    const int b2_box = pair ? BN / 2 : BN;
    CUtensorMap mA1, mB1, mB3, mA2, mB2;
    if (!make_map_bf16(&mA1, a.xe, R, a.d, BM) || !make_map_bf16(&mB1, a.w1, (int64_t)a.N * a.d_ff, a.d, b1_box) ||
        !make_map_bf16(&mA2, a.h, R, a.d_ff, BM) ||
        (!a.stage1_only && !make_map_bf16(&mB2, a.w2, (int64_t)a.N * a.d, a.d_ff, b2_box)))
        return cudaErrorInvalidValue;
    if (swiglu) {
        if (!make_map_bf16(&mB3, a.w3, (int64_t)a.N * a.d_ff, a.d, b1_box)) return cudaErrorInvalidValue;
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
    p1.pre_out = reinterpret_cast<__nv_bfloat16*>(a.pre_out);
    CUtensorMap mO1, mO2;   // the compact outputs H [R, d_ff] and ye [R, d], 32-row boxes (TMA stores)
    if (!make_map_bf16(&mO1, a.h, R, a.d_ff, 32)) return cudaErrorInvalidValue;
    cudaError_t err = swiglu ? run_gemm_any<EPI_SWIGLU>(mA1, mB1, mB3, mO1, p1, s)
                             : run_gemm_any<EPI_RELU>(mA1, mB1, mB3, mO1, p1, s);
    if (err != cudaSuccess || a.stage1_only) return err;
    if (a.mid_event && (err = cudaEventRecord((cudaEvent_t)a.mid_event, s)) != cudaSuccess) return err;

    GemmParams p2{};
    p2.offsets = a.offsets;
    p2.N = a.N;
    p2.n_dim = a.d;
    p2.k_dim = a.d_ff;
    p2.out_ld = a.d;
    p2.bias = reinterpret_cast<const __nv_bfloat16*>(a.b2);
    p2.status = &a.hdr->status;
    p2.reverse = 1;
    p2.limit_ns = kWaitLimitNs;
    if (a.scatter_out || a.scatter_ptrs) {
        p2.out = reinterpret_cast<__nv_bfloat16*>(a.scatter_out);
        p2.row_token = a.row_token;
        p2.row_gate = a.row_gate;
        p2.out_ptrs = a.scatter_ptrs;
        p2.row_rank = a.row_rank;
        return run_gemm_any<EPI_SCATTER>(mA2, mB2, mB2, mA2, p2, s);
    }
    p2.out = reinterpret_cast<__nv_bfloat16*>(a.ye);
    if (!make_map_bf16(&mO2, a.ye, R, a.d, 32)) return cudaErrorInvalidValue;
    return run_gemm_any<EPI_BIAS>(mA2, mB2, mB2, mO2, p2, s);
}

}  // namespace moe
