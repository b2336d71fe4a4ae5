// Capacity-limited dispatch of the MoE layer: slot claiming in token order,
// drop mask, compact expert-major row map and the gather of x into it.
//
// Definition: CS25 Lecture 05 notes "Scaling Transformers through Sparsity",
// section "Static compilation meets dynamic routing" (capacity-aware dispatch:
// in token order a token joins its expert's slots while fewer than C are taken,
// otherwise it skips the expert); CMU 10-423 Lecture 16, section 6.1 (GShard
// rule: every token's first choice is placed before any second choice); "From
// Switch Transformer to GLaM", "Expert Capacity and Token Dropping".
//
// pos[t, r] = number of earlier claims on idx[t, r], where "earlier" is
// rank-major then token order; an assignment is kept iff pos < C.  This is an
// exclusive prefix count over (rank, token) per expert, computed as:
//   1. scan_kernel: a block owns 1024 consecutive tokens.  Warps rank their
//      32-token groups with __match_any_sync (tokens of a warp that pick the same
//      expert), giving in-block ranks and a per-(rank, expert) block aggregate;
//      a decoupled look-back across blocks (dynamic block tickets, bounded
//      spin) turns the aggregates into exclusive block prefixes.  The last block
//      to finish derives counts, kept = min(count, C) and the offsets.
//   2. scatter_kernel: per assignment, adds the rank-0 total to rank-1
//      positions, writes pos/drop and the row map, and copies x[t] into its
//      compact row with 16-byte vector accesses (a warp per eight assignments).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kScanThreads = 256;
constexpr int kWarpTokens = kScanTokens / 8;   // kScanTokens (common.cuh) = 8 warps x 128 tokens
constexpr uint32_t kFlagAgg = 1u << 30;    // block aggregate published
constexpr uint32_t kFlagPre = 2u << 30;    // inclusive prefix published
constexpr uint32_t kValMask = (1u << 30) - 1u;

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Decoupled look-back for one counter: publish this block's aggregate, then walk
// back over predecessors until one with an inclusive prefix is found.  The
// predecessors' states are read kLookWindow at a time (independent loads, one
// memory round trip per window instead of one per predecessor: all blocks
// publish their aggregates at about the same time, so a late block would
// otherwise walk half its predecessors one load after another) and consumed in
// order.  Waiting on a predecessor that has not published is bounded by
// limit_ns; on expiry the wait latches MOE_ERR_TIMEOUT and this block publishes
// anyway, so successors never wait on it.
constexpr int kLookWindow = 16;
__device__ uint32_t lookback(uint32_t* state, int bid, int c, int kN, uint32_t agg,
                             long long limit_ns, int32_t* status) {
    if (bid == 0) {
        st_relaxed(state + c, kFlagPre | agg);
        return 0u;
    }
    st_relaxed(state + (int64_t)bid * kN + c, kFlagAgg | agg);
    uint32_t excl = 0;
    int p = bid - 1;   // the next predecessor not yet added
    long long t_start = -1;
    unsigned spins = 0;
    bool found = false;
    while (!found) {
        uint32_t v[kLookWindow];
#pragma unroll
        for (int j = 0; j < kLookWindow; ++j)   // block 0 always ends the walk, so p - j < 0 is never consumed
            v[j] = p - j >= 0 ? ld_relaxed(state + (int64_t)(p - j) * kN + c) : kFlagPre;
        int used = 0;
#pragma unroll
        for (int j = 0; j < kLookWindow; ++j) {
            const uint32_t fl = v[j] & ~kValMask;
            if (fl == 0u) break;   // not published yet: the next window starts here
            excl += v[j] & kValMask;
            ++used;
            if (fl == kFlagPre) {
                found = true;
                break;
            }
        }
        if (found) break;
        p -= used;
        if (used == 0) {   // the nearest unread predecessor has not published yet
            if (t_start < 0) t_start = global_ns();
            if ((++spins & 63u) == 0u && global_ns() - t_start > limit_ns) {
                latch_status(status, MOE_ERR_TIMEOUT);
                break;
            }
            __nanosleep(64);
        }
    }
    st_relaxed(state + (int64_t)bid * kN + c, kFlagPre | ((excl + agg) & kValMask));
    return excl;
}

__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const int32_t* __restrict__ idx, int64_t T, int N, int k, int C, int nblk,
            const int32_t* __restrict__ claim_base, int32_t* __restrict__ pos, int32_t* __restrict__ counts,
            int32_t* __restrict__ kept, int32_t* __restrict__ offsets, uint32_t* __restrict__ state, WsHeader* hdr,
            long long limit_ns) {
    pdl_wait();
    pdl_launch();
    __shared__ int s_bid;
    __shared__ int s_last;
    __shared__ int s_wcnt[8][256];
    __shared__ uint32_t s_excl[256];
    __shared__ int s_tot[256];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kN = k * N;
    if (tid == 0) s_bid = atomicAdd(&hdr->scan_ticket, 1);
    for (int q = tid; q < 8 * 256; q += kScanThreads) (&s_wcnt[0][0])[q] = 0;
    __syncthreads();
    const int bid = s_bid;
    const int64_t tw0 = (int64_t)bid * kScanTokens + warp * kWarpTokens;

    // 1. in-warp ranks, in token order, per (rank, expert) counter; the warp's
    //    choices are loaded first, all at once (one memory round trip)
    int keys[kWarpTokens / 32][2];
#pragma unroll
    for (int it = 0; it < kWarpTokens / 32; ++it) {
        const int64_t t = tw0 + it * 32 + lane;
#pragma unroll
        for (int r = 0; r < 2; ++r) keys[it][r] = (r < k && t < T) ? r * N + idx[t * k + r] : -1;
    }
    int rank[kWarpTokens / 32][2];
    const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int it = 0; it < kWarpTokens / 32; ++it) {
        const int64_t t = tw0 + it * 32 + lane;
        const bool valid = t < T;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            if (r >= k) break;
            const int key = keys[it][r];
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            const int before = __popc(peers & lt_mask);
            if (valid) rank[it][r] = s_wcnt[warp][key] + before;
            __syncwarp();
            if (valid && lane == __ffs(peers) - 1) s_wcnt[warp][key] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();

    // 2. per counter: warp offsets inside the block, block aggregate, look-back
    for (int c = tid; c < kN; c += kScanThreads) {
        int run = 0;
        for (int w = 0; w < 8; ++w) {
            int v = s_wcnt[w][c];
            s_wcnt[w][c] = run;
            run += v;
        }
        s_excl[c] = lookback(state, bid, c, kN, (uint32_t)run, limit_ns, &hdr->status);
    }
    __syncthreads();

    // 3. local claim numbers (rank 1 still lacks the global rank-0 total)
#pragma unroll
    for (int it = 0; it < kWarpTokens / 32; ++it) {
        const int64_t t = tw0 + it * 32 + lane;
        if (t >= T) break;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            if (r >= k) break;
            const int key = keys[it][r];
            pos[t * k + r] = (int)s_excl[key] + s_wcnt[warp][key] + rank[it][r];
        }
    }

    // 4. the last block to finish derives counts, kept and offsets
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&hdr->scan_done, 1) == nblk - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int c = tid; c < kN; c += kScanThreads) {
        int tot = (int)(ld_relaxed(state + (int64_t)(nblk - 1) * kN + c) & kValMask);
        s_tot[c] = tot;
        counts[c] = tot;
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int e = 0; e < N; ++e) {
            // this shard's kept claims: rank-0 claims numbered from base0, rank-1
            // claims from base1 (after every rank-0 claim); a whole batch is one
            // shard with base0 = 0 and base1 = its own rank-0 total
            const int c0 = s_tot[e], c1 = k == 2 ? s_tot[N + e] : 0;
            const int base0 = claim_base ? claim_base[e] : 0;
            const int base1 = claim_base ? claim_base[N + e] : c0;
            const int ke = kept_after(base0, c0, C) + (k == 2 ? kept_after(base1, c1, C) : 0);
            kept[e] = ke;
            offsets[e] = acc;
            acc += ke;
        }
        offsets[N] = acc;
    }
}

// Slot bookkeeping of one assignment a (claim order: position q, rank r):
// writes pos / drop and, when kept, the row map; returns the compact row, or -1
// when the assignment is dropped.  t receives the token.
__device__ __forceinline__ int claim_slot(int64_t a, const int32_t* __restrict__ idx, const float* __restrict__ gate,
                                          int N, int k, int C, const int32_t* __restrict__ claim_base,
                                          int32_t* __restrict__ pos, uint8_t* __restrict__ drop,
                                          const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                                          int32_t* __restrict__ row_token, float* __restrict__ row_gate,
                                          const int32_t* __restrict__ perm, const int32_t* __restrict__ pos_in,
                                          int64_t& t) {
    // Batch priority: the token at position q is perm[q], and the scan's claim
    // numbers are in pos_in (claim-order layout).
    const int64_t q = a / k;
    const int r = (int)(a - q * k);
    t = perm ? (int64_t)perm[q] : q;
    const int64_t ao = t * k + r;   // the assignment in token order
    const int e = idx[ao];
    const int lp = pos_in ? pos_in[a] : pos[a];   // claim number among this shard's rank-r claims on e
    int p, row_off;
    if (r == 0) {
        p = (claim_base ? claim_base[e] : 0) + lp;
        row_off = lp;
    } else {   // every rank-0 claim precedes the rank-1 claims
        const int base0 = claim_base ? claim_base[e] : 0;
        p = (claim_base ? claim_base[N + e] : counts[e]) + lp;
        row_off = kept_after(base0, counts[e], C) + lp;
    }
    const bool keep = p < C;
    pos[ao] = p;
    drop[ao] = keep ? 0 : 1;
    if (!keep) return -1;
    const int row = offsets[e] + row_off;
    row_token[row] = (int32_t)t;
    row_gate[row] = gate[ao];
    return row;
}

// One warp per kScatterRows consecutive assignments: lanes 0 .. kScatterRows-1
// do the slot bookkeeping of one assignment each (one dependent chain of loads
// per warp instead of one per row), then the warp moves the rows two at a
// time -- a kept row's x[t] into its compact row, a dropped token's output row
// set to zero when zero_out is given -- with up to 2 x kCopyUnroll 16-byte
// loads per lane in flight.  At Switch-Base sizes that is 1024 blocks of 256
// threads (about two waves); with one assignment per warp, 8192 blocks each
// living about a microsecond were bound by block launches.
constexpr int kScatterRows = 8;
constexpr int kCopyUnroll = 4;

template <typename XT>
__global__ void __launch_bounds__(256)
scatter_kernel(const XT* __restrict__ x, const int32_t* __restrict__ idx, const float* __restrict__ gate,
               int64_t T, int d, int N, int k, int C,
               const int32_t* __restrict__ claim_base, int32_t* __restrict__ pos, uint8_t* __restrict__ drop,
               const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets, int32_t* __restrict__ row_token,
               float* __restrict__ row_gate, XT* __restrict__ xe, XT* __restrict__ zero_out, const AuxArgs aux,
               const int32_t* __restrict__ perm, const int32_t* __restrict__ pos_in) {
    pdl_wait();
    pdl_launch();
    // the extra block (the first, so it is scheduled at once and runs beside
    // the row copies): load-balancing loss from the router's partials
    if (aux.G > 0 && blockIdx.x == 0) {
        __shared__ double s_aux[kAuxScratch];
        aux_reduce_block(aux, s_aux);
        return;
    }
    const int lane = threadIdx.x & 31;
    const int64_t n_assign = T * k;
    const int64_t a0 = ((int64_t)(blockIdx.x - (aux.G > 0 ? 1 : 0)) * 8 + (threadIdx.x >> 5)) * kScatterRows;
    if (a0 >= n_assign) return;
    // per lane i < kScatterRows: what happens to assignment a0 + i's row --
    // >= 0 copy x[t] to that compact row, -1 zero out[t], -2 nothing
    int act = -2;
    int64_t t = 0;
    if (lane < kScatterRows && a0 + lane < n_assign) {
        const int row = claim_slot(a0 + lane, idx, gate, N, k, C, claim_base, pos, drop, counts, offsets, row_token,
                                   row_gate, perm, pos_in, t);
        act = row >= 0 ? (xe != nullptr ? row : -2) : (zero_out != nullptr ? -1 : -2);
    }
    const size_t bytes = (size_t)d * sizeof(XT);
    const uint4 z4 = make_uint4(0, 0, 0, 0);
#pragma unroll 1
    for (int i = 0; i < kScatterRows; i += 2) {
        const int act0 = __shfl_sync(0xffffffffu, act, i), act1 = __shfl_sync(0xffffffffu, act, i + 1);
        const int64_t t0 = __shfl_sync(0xffffffffu, t, i), t1 = __shfl_sync(0xffffffffu, t, i + 1);
        if (act0 == -2 && act1 == -2) continue;
        const XT* s0 = x + t0 * (int64_t)d;
        const XT* s1 = x + t1 * (int64_t)d;
        XT* d0 = act0 >= 0 ? xe + (int64_t)act0 * d : (act0 == -1 ? zero_out + t0 * (int64_t)d : nullptr);
        XT* d1 = act1 >= 0 ? xe + (int64_t)act1 * d : (act1 == -1 ? zero_out + t1 * (int64_t)d : nullptr);
        if (bytes % 16 == 0) {
            const char* c0 = reinterpret_cast<const char*>(s0);
            const char* c1 = reinterpret_cast<const char*>(s1);
            char* e0 = reinterpret_cast<char*>(d0);
            char* e1 = reinterpret_cast<char*>(d1);
            for (size_t o = (size_t)lane * 16; o < bytes; o += 32 * 16 * kCopyUnroll) {
                uint4 v0[kCopyUnroll], v1[kCopyUnroll];
#pragma unroll
                for (int u = 0; u < kCopyUnroll; ++u) {
                    const size_t oo = o + (size_t)u * 32 * 16;
                    v0[u] = (act0 >= 0 && oo < bytes) ? __ldg(reinterpret_cast<const uint4*>(c0 + oo)) : z4;
                    v1[u] = (act1 >= 0 && oo < bytes) ? __ldg(reinterpret_cast<const uint4*>(c1 + oo)) : z4;
                }
#pragma unroll
                for (int u = 0; u < kCopyUnroll; ++u) {
                    const size_t oo = o + (size_t)u * 32 * 16;
                    if (oo < bytes) {
                        if (e0) *reinterpret_cast<uint4*>(e0 + oo) = v0[u];
                        if (e1) *reinterpret_cast<uint4*>(e1 + oo) = v1[u];
                    }
                }
            }
        } else {
            for (int j = lane; j < d; j += 32) {
                if (d0) d0[j] = act0 >= 0 ? s0[j] : XT(0.f);
                if (d1) d1[j] = act1 >= 0 ? s1[j] : XT(0.f);
            }
        }
    }
}

// The same slot bookkeeping without the compact copy and without output rows
// to zero (moe_dispatch called with no xe): one thread per assignment writes
// pos, drop, row_token and row_gate.
__global__ void __launch_bounds__(256)
rowmap_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, int64_t T, int N, int k, int C,
              const int32_t* __restrict__ claim_base, int32_t* __restrict__ pos, uint8_t* __restrict__ drop,
              const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
              int32_t* __restrict__ row_token, float* __restrict__ row_gate, const AuxArgs aux,
              const int32_t* __restrict__ perm, const int32_t* __restrict__ pos_in) {
    pdl_wait();
    pdl_launch();
    if (aux.G > 0 && blockIdx.x == 0) {   // the load-balancing loss, as in scatter_kernel
        __shared__ double s_aux[kAuxScratch];
        aux_reduce_block(aux, s_aux);
        return;
    }
    const int64_t a = (int64_t)(blockIdx.x - (aux.G > 0 ? 1 : 0)) * 256 + threadIdx.x;
    if (a >= T * k) return;
    int64_t t;
    claim_slot(a, idx, gate, N, k, C, claim_base, pos, drop, counts, offsets, row_token, row_gate, perm, pos_in, t);
}

// ---- batch priority: the claim order --------------------------------------
// CS25 Lecture 05 notes, section on Vision MoE: with capacity short, priority
// routing lets the tokens with the highest priority score take the expert
// slots first.  The score is the token's first-choice gate; the claim order is
// descending score, ties to the lower token index (rank-major as before).
// Key: 0xFFFFFFFF - bits(gate) (gates are >= 0, so their bit patterns order
// like their values), ascending.  The batch's key range [kmin, kmax] is cut
// into kPrioBuckets equal intervals (a monotone bucket map).  A token's place
// in the order is the number of tokens in lower buckets plus, within its
// bucket, the number of tokens with a smaller key or the same key and a lower
// index -- exact and independent of the order in which the bucket lists were
// filled.  Cost: one pass per token over its bucket (quadratic only when most
// scores fall into one interval, e.g. many equal scores).
__device__ __forceinline__ uint32_t prio_key(const float* gate, int64_t t, int k) {
    return 0xFFFFFFFFu - __float_as_uint(gate[t * k]);
}
// range[0] = kmin, range[1] = kmax of the batch
__device__ __forceinline__ uint32_t prio_bucket(uint32_t key, const uint32_t* range) {
    const uint32_t lo = range[0], width = ((range[1] - lo) >> 16) + 1u;
    return (key - lo) / width;   // < kPrioBuckets
}

__global__ void __launch_bounds__(256)
prio_range_kernel(const float* __restrict__ gate, int64_t T, int k, uint32_t* __restrict__ range) {
    pdl_wait();
    pdl_launch();
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t u = prio_key(gate, t, k);
        mn = min(mn, u);
        mx = max(mx, u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMin(&range[0], mn);
        atomicMax(&range[1], mx);
    }
}

__global__ void __launch_bounds__(256)
prio_hist_kernel(const float* __restrict__ gate, int64_t T, int k, const uint32_t* __restrict__ range,
                 int32_t* __restrict__ hist) {
    pdl_wait();
    pdl_launch();
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x)
        atomicAdd(&hist[prio_bucket(prio_key(gate, t, k), range)], 1);
}

// exclusive prefix of the kPrioBuckets counts, in place; hist[kPrioBuckets] = T.
// One block of 32 warps; warp w owns the contiguous chunk [w C, (w + 1) C) and
// scans it 32 entries at a time (coalesced), carrying the running total.
__global__ void __launch_bounds__(1024) prio_scan_kernel(int32_t* __restrict__ hist) {
    pdl_wait();
    pdl_launch();
    __shared__ int32_t s_warp[32];
    constexpr int CHUNK = kPrioBuckets / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t* h = hist + warp * CHUNK;
    int32_t tot = 0;
    for (int j = lane; j < CHUNK; j += 32) tot += h[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if (lane == 0) s_warp[warp] = tot;
    __syncthreads();
    int32_t carry = 0;
    for (int w = 0; w < warp; ++w) carry += s_warp[w];
    for (int j0 = 0; j0 < CHUNK; j0 += 32) {
        const int32_t c = h[j0 + lane];
        int32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        h[j0 + lane] = carry + incl - c;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (threadIdx.x == 1023) hist[kPrioBuckets] = carry;
}

// bucket lists: list[base[b] + n] = t, n in arrival order
__global__ void __launch_bounds__(256)
prio_fill_kernel(const float* __restrict__ gate, int64_t T, int k, const uint32_t* __restrict__ range,
                 const int32_t* __restrict__ base, int32_t* __restrict__ cursor, int32_t* __restrict__ list) {
    pdl_wait();
    pdl_launch();
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t b = prio_bucket(prio_key(gate, t, k), range);
        list[base[b] + atomicAdd(&cursor[b], 1)] = (int32_t)t;
    }
}

// place of t in the claim order; perm[place] = t, idx_sorted[place] = idx[t]
__global__ void __launch_bounds__(256)
prio_rank_kernel(const float* __restrict__ gate, const int32_t* __restrict__ idx, int64_t T, int k,
                 const uint32_t* __restrict__ range, const int32_t* __restrict__ base,
                 const int32_t* __restrict__ list, int32_t* __restrict__ perm, int32_t* __restrict__ idx_sorted) {
    pdl_wait();
    pdl_launch();
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t u = prio_key(gate, t, k);
        const uint32_t b = prio_bucket(u, range);
        const int32_t lo = base[b], hi = base[b + 1];
        int32_t c = 0;
        for (int32_t j = lo; j < hi; ++j) {
            const int64_t t2 = list[j];
            const uint32_t u2 = prio_key(gate, t2, k);
            c += (u2 < u || (u2 == u && t2 < t)) ? 1 : 0;
        }
        const int64_t place = (int64_t)lo + c;
        perm[place] = (int32_t)t;
        for (int r = 0; r < k; ++r) idx_sorted[place * k + r] = idx[t * k + r];
    }
}

// ---- No-Token-Left-Behind re-routing (top-1) --------------------------------
// CS25 Lecture 05 notes, "No Token Left Behind": a token whose expert is full
// goes on to its second, third ... choice until it gets a slot.  Stage s: each
// token still without a slot claims, in token order, on its (s+1)-th expert
// (router probabilities descending, ties to the lower index), numbered after
// every claim already made on that expert; kept iff that number is below C.
//
// One cooperative launch runs every stage (its blocks are co-resident, so they
// may wait on one another).  Block b owns the contiguous tokens [b TB, (b+1) TB).
// Per stage: (1) each block picks the next expert of its unplaced tokens and
// ranks them per expert in token order (warp match + running counts over
// 1024-token pieces), and publishes its per-expert claim counts; (2) one grid
// barrier; (3) every block sums the counts of the blocks before it (exclusive
// prefix) and of all blocks (the stage's claims), places its tokens whose claim
// number claims_before[e] + prefix[e] + rank is below C, and publishes how many
// of its tokens are still unplaced.  The next stage's barrier makes those counts
// visible: when none is left, every block stops (the remaining stages would
// claim nothing).  Dropped tokens then report their first choice with pos = C,
// and block 0 writes counts / kept / offsets.  Scratch is double-buffered by
// stage parity, so a block never overwrites counts a slower block still reads.

// expert a (probability pa) comes before expert b in a token's order
__device__ __forceinline__ bool ntlb_before(float pa, int a, float pb, int b) {
    return pa > pb || (pa == pb && a < b);
}

// The first expert after `le` (probability lpv) in the token's order; le < 0:
// the token's first choice.
__device__ __forceinline__ int ntlb_next(const float* __restrict__ p, int N, int le, float lpv) {
    int best = -1;
    float bp = 0.f;
    for (int e = 0; e < N; ++e) {
        const float pe = __ldg(p + e);
        if (le >= 0 && !ntlb_before(lpv, le, pe, e)) continue;
        if (best < 0 || ntlb_before(pe, e, bp, best)) {
            best = e;
            bp = pe;
        }
    }
    return best;
}

struct NtlbGrid {
    const float* probs; int64_t T; int N; int C; int64_t TB;
    int32_t* expert; float* gate; int32_t* pos;
    int32_t* counts; int32_t* kept; int32_t* offsets;
    int32_t* ch; int32_t* last; int32_t* first; int32_t* placed; int32_t* lp;
    int32_t* agg;        // [2][gridDim.x][N] per-block claims of the stage
    int32_t* unplaced;   // [2][gridDim.x]
    uint32_t* bar;       // grid barrier arrivals (0 at launch)
    int32_t* status;
    long long limit_ns;
};

// Grid-wide barrier of a cooperative launch (bounded: on expiry the status is
// latched and false returned, and the caller stops).
__device__ bool ntlb_grid_sync(uint32_t* bar, uint32_t target, long long limit_ns, int32_t* status, int* s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(bar, 1u);
        const long long t0 = global_ns();
        int ok = 1;
        for (unsigned i = 0; ld_relaxed(bar) < target; ++i) {
            if ((i & 63u) == 63u && global_ns() - t0 > limit_ns) {
                latch_status(status, MOE_ERR_TIMEOUT);
                ok = 0;
                break;
            }
        }
        __threadfence();
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

__global__ void __launch_bounds__(kScanThreads) ntlb_grid_kernel(const NtlbGrid a) {
    pdl_wait();
    pdl_launch();
    __shared__ int32_t s_claims[128];      // claims on each expert before this stage
    __shared__ int32_t s_cnt[128];         // this block's claims in this stage, so far
    __shared__ int32_t s_base[128];        // s_cnt before the current 1024-token piece
    __shared__ int32_t s_wcnt[8][128];     // per warp, then per-warp exclusive offsets
    __shared__ int32_t s_excl[128];        // claims of earlier blocks in this stage
    __shared__ int32_t s_red[kScanThreads / 32];
    __shared__ int s_ok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.N, G = (int)gridDim.x, b = (int)blockIdx.x;
    const int64_t t_lo = (int64_t)b * a.TB;
    const int64_t t_hi = min(a.T, t_lo + a.TB);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int e = tid; e < N; e += kScanThreads) {
        s_claims[e] = 0;
        s_cnt[e] = 0;
    }
    for (int q = tid; q < 8 * 128; q += kScanThreads) (&s_wcnt[0][0])[q] = 0;
    __syncthreads();
    uint32_t nbar = 0;
    bool ok = true;
    for (int s = 0; s < N && ok; ++s) {
        const int par = s & 1;
        // (1) next choice and the rank among this block's claims on it, token order
        for (int64_t base = t_lo; base < t_hi; base += kScanTokens) {
            int rk[kWarpTokens / 32], ex[kWarpTokens / 32];
#pragma unroll
            for (int it = 0; it < kWarpTokens / 32; ++it) {
                const int64_t t = base + warp * kWarpTokens + it * 32 + lane;
                int e = -1;
                if (t < t_hi) {
                    const float* p = a.probs + t * N;
                    if (s == 0) {
                        e = ntlb_next(p, N, -1, 0.f);
                        a.placed[t] = 0;
                        a.first[t] = e;
                        a.last[t] = e;
                    } else if (!a.placed[t]) {
                        const int le = a.last[t];
                        e = ntlb_next(p, N, le, __ldg(p + le));   // s < N: an untried expert is left
                        a.last[t] = e;
                    }
                    a.ch[t] = e;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, e);
                ex[it] = e;
                rk[it] = e >= 0 ? s_wcnt[warp][e] + __popc(peers & lt_mask) : 0;
                __syncwarp();
                if (e >= 0 && lane == __ffs(peers) - 1) s_wcnt[warp][e] += __popc(peers);
                __syncwarp();
            }
            __syncthreads();
            for (int e = tid; e < N; e += kScanThreads) {   // warp offsets inside the piece
                int run = s_cnt[e];
                s_base[e] = run;
                for (int w = 0; w < 8; ++w) {
                    const int v = s_wcnt[w][e];
                    s_wcnt[w][e] = run;
                    run += v;
                }
                s_cnt[e] = run;
            }
            __syncthreads();
#pragma unroll
            for (int it = 0; it < kWarpTokens / 32; ++it) {
                const int64_t t = base + warp * kWarpTokens + it * 32 + lane;
                if (t < t_hi && ex[it] >= 0) a.lp[t] = s_wcnt[warp][ex[it]] + rk[it];
            }
            __syncthreads();
            for (int q = tid; q < 8 * N; q += kScanThreads) s_wcnt[q / N][q % N] = 0;
            __syncthreads();
        }
        for (int e = tid; e < N; e += kScanThreads) {
            a.agg[((int64_t)par * G + b) * N + e] = s_cnt[e];
            s_cnt[e] = 0;
        }
        // (2) every block's counts of this stage (and unplaced counts of the last) are visible
        nbar += (uint32_t)G;
        if (!ntlb_grid_sync(a.bar, nbar, a.limit_ns, a.status, &s_ok)) {
            ok = false;
            break;
        }
        if (s > 0) {   // nothing was left unplaced after the previous stage: done
            int left = 0;
            for (int q = tid; q < G; q += kScanThreads) left += __ldcg(a.unplaced + (int64_t)(par ^ 1) * G + q);
            left = __syncthreads_or(left != 0);
            if (!left) break;
        }
        // (3) claim numbers and placement
        for (int e = tid; e < N; e += kScanThreads) {
            int ex_ = 0, tot = 0;
            const int32_t* col = a.agg + (int64_t)par * G * N + e;
            for (int q = 0; q < G; ++q) {
                const int v = __ldcg(col + (int64_t)q * N);
                ex_ += q < b ? v : 0;
                tot += v;
            }
            s_excl[e] = ex_;
            s_base[e] = tot;
        }
        __syncthreads();
        int left = 0;
        for (int64_t t = t_lo + tid; t < t_hi; t += kScanThreads) {
            if (a.placed[t]) continue;
            const int e = a.ch[t];
            const int64_t c = (int64_t)s_claims[e] + s_excl[e] + a.lp[t];
            if (c < (int64_t)a.C) {
                a.placed[t] = 1;
                a.expert[t] = e;
                a.pos[t] = (int32_t)c;
                a.gate[t] = a.probs[t * N + e];
            } else {
                ++left;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) left += __shfl_xor_sync(0xffffffffu, left, o);
        if (lane == 0) s_red[warp] = left;
        __syncthreads();
        if (tid == 0) {
            int sum = 0;
            for (int w = 0; w < kScanThreads / 32; ++w) sum += s_red[w];
            a.unplaced[(int64_t)par * G + b] = sum;
        }
        for (int e = tid; e < N; e += kScanThreads) s_claims[e] += s_base[e];
        __syncthreads();
    }
    if (!ok) return;
    // dropped: first choice, claim number C
    for (int64_t t = t_lo + tid; t < t_hi; t += kScanThreads) {
        if (a.placed[t]) continue;
        const int e = a.first[t];
        a.expert[t] = e;
        a.pos[t] = a.C;
        a.gate[t] = a.probs[t * N + e];
    }
    if (b == 0 && tid == 0) {   // every block holds the same claim totals
        int32_t acc = 0;
        for (int e = 0; e < N; ++e) {
            const int32_t c = s_claims[e];
            a.counts[e] = c;
            a.kept[e] = c < a.C ? c : a.C;
            a.offsets[e] = acc;
            acc += a.kept[e];
        }
        a.offsets[N] = acc;
    }
}

// Claims per (rank, expert) of this shard: counts[r][e] (int atomics, so the
// result is exact and order-independent).
__global__ void __launch_bounds__(256)
count_kernel(const int32_t* __restrict__ idx, int64_t T, int N, int k, int32_t* __restrict__ counts) {
    __shared__ int h[256];
    for (int c = threadIdx.x; c < k * N; c += blockDim.x) h[c] = 0;
    __syncthreads();
    const int64_t n = T * k;
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < n; a += (int64_t)gridDim.x * blockDim.x)
        atomicAdd(&h[(int)(a % k) * N + idx[a]], 1);
    __syncthreads();
    for (int c = threadIdx.x; c < k * N; c += blockDim.x)
        if (h[c]) atomicAdd(&counts[c], h[c]);
}

// Claim base of shard `shard` from every shard's counts [S][k][N]:
//   base[0][e] = rank-0 claims on e by shards before this one;
//   base[1][e] = all shards' rank-0 claims on e + rank-1 claims by earlier shards.
__global__ void claim_base_kernel(const int32_t* __restrict__ all, int S, int shard, int k, int N,
                                  int32_t* __restrict__ base) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= N) return;
    int b0 = 0, tot0 = 0, b1 = 0;
    for (int s = 0; s < S; ++s) {
        const int c0 = all[(int64_t)s * k * N + e];
        tot0 += c0;
        if (s < shard) {
            b0 += c0;
            if (k == 2) b1 += all[(int64_t)s * k * N + N + e];
        }
    }
    base[e] = b0;
    if (k == 2) base[N + e] = tot0 + b1;
}

// Load-balancing loss over shards: f and P are token-weighted means of the
// shards' f_s and P_s (fp64, shard order), aux = alpha N sum_i f_i P_i.
__global__ void aux_shards_kernel(int S, int N, const int64_t* __restrict__ tokens, const double* __restrict__ f_all,
                                  const double* __restrict__ P_all, float alpha, double* __restrict__ f,
                                  double* __restrict__ P, double* __restrict__ aux) {
    __shared__ double fp[128];
    const int e = threadIdx.x;
    double T = 0.0;
    for (int s = 0; s < S; ++s) T += (double)tokens[s];
    if (e < N) {
        double fs = 0.0, ps = 0.0;
        for (int s = 0; s < S; ++s) {
            fs += (double)tokens[s] * f_all[(int64_t)s * N + e];
            ps += (double)tokens[s] * P_all[(int64_t)s * N + e];
        }
        const double fe = T > 0 ? fs / T : 0.0, pe = T > 0 ? ps / T : 0.0;
        if (f) f[e] = fe;
        if (P) P[e] = pe;
        fp[e] = fe * pe;
    }
    __syncthreads();
    if (e == 0 && aux) {
        double acc = 0.0;
        for (int q = 0; q < N; ++q) acc += fp[q];
        *aux = (double)alpha * (double)N * acc;
    }
}

// Test hook: one block whose predecessor (block 0) never publishes.
__global__ void lookback_probe_kernel(uint32_t* state, WsHeader* hdr, long long limit_ns) {
    if (threadIdx.x < 4) lookback(state, 1, threadIdx.x, 4, 1u, limit_ns, &hdr->status);
}

}  // namespace

int scan_blocks(int64_t T) { return (int)((T + kScanTokens - 1) / kScanTokens); }

// blocks of scatter_kernel: 8 warps of kScatterRows assignments, plus the aux block
static unsigned scatter_grid(int64_t n_assign, bool aux_block) {
    return (unsigned)((n_assign + 8 * kScatterRows - 1) / (8 * kScatterRows)) + (aux_block ? 1u : 0u);
}

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s) {
    const int nblk = scan_blocks(a.T);
    if (nblk == 0) return cudaSuccess;
    cudaError_t err;
    // claim order: token order, or batch priority (the scan then runs over the
    // expert choices in claim order and the gather maps back through perm)
    const int32_t* scan_idx = a.idx;
    int32_t* scan_pos = a.pos;
    const int32_t* perm = nullptr;
    const int32_t* pos_in = nullptr;
    if (a.prio.perm) {
        const PrioArgs& q = a.prio;
        if ((err = cudaMemsetAsync(q.hist, 0, sizeof(int32_t) * (kPrioBuckets + 1), s)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(q.cursor, 0, sizeof(int32_t) * kPrioBuckets, s)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(q.range, 0xFF, sizeof(uint32_t), s)) != cudaSuccess) return err;     // kmin
        if ((err = cudaMemsetAsync(q.range + 1, 0, sizeof(uint32_t), s)) != cudaSuccess) return err;   // kmax
        const unsigned pg = (unsigned)((a.T + 255) / 256 < 4096 ? (a.T + 255) / 256 : 4096);
        if ((err = launch_k(prio_range_kernel, dim3(pg), dim3(256), 0, s, 1, a.gate, a.T, a.k, q.range)) != cudaSuccess)
            return err;
        if ((err = launch_k(prio_hist_kernel, dim3(pg), dim3(256), 0, s, 1, a.gate, a.T, a.k,
                            static_cast<const uint32_t*>(q.range), q.hist)) != cudaSuccess)
            return err;
        if ((err = launch_k(prio_scan_kernel, dim3(1), dim3(1024), 0, s, 1, q.hist)) != cudaSuccess) return err;
        if ((err = launch_k(prio_fill_kernel, dim3(pg), dim3(256), 0, s, 1, a.gate, a.T, a.k,
                            static_cast<const uint32_t*>(q.range), static_cast<const int32_t*>(q.hist), q.cursor,
                            q.list)) != cudaSuccess)
            return err;
        if ((err = launch_k(prio_rank_kernel, dim3(pg), dim3(256), 0, s, 1, a.gate, a.idx, a.T, a.k,
                            static_cast<const uint32_t*>(q.range), static_cast<const int32_t*>(q.hist),
                            static_cast<const int32_t*>(q.list), q.perm, q.idx_sorted)) != cudaSuccess)
            return err;
        scan_idx = q.idx_sorted;
        scan_pos = q.pos_sorted;
        perm = q.perm;
        pos_in = q.pos_sorted;
    }
    // fresh tickets and look-back flags for this call
    err = cudaMemsetAsync(&a.hdr->scan_ticket, 0, 2 * sizeof(int32_t), s);
    if (err != cudaSuccess) return err;
    err = cudaMemsetAsync(a.scan_state, 0, sizeof(uint32_t) * (size_t)nblk * a.k * a.N, s);
    if (err != cudaSuccess) return err;
    err = launch_k(scan_kernel, dim3((unsigned)nblk), dim3(kScanThreads), 0, s, 1, scan_idx, a.T, a.N, a.k, a.C, nblk,
                   a.claim_base, scan_pos, a.counts, a.kept, a.offsets, a.scan_state, a.hdr, kWaitLimitNs);
    if (err != cudaSuccess) return err;
    if (a.xe == nullptr && a.zero_out == nullptr) {   // row map only: thread per assignment
        const unsigned grid = (unsigned)((a.T * a.k + 255) / 256) + (a.aux.G > 0 ? 1u : 0u);
        return launch_k(rowmap_kernel, dim3(grid), dim3(256), 0, s, 1, a.idx, a.gate, a.T, a.N, a.k, a.C,
                        a.claim_base, a.pos, a.drop, a.counts, a.offsets, a.row_token, a.row_gate, a.aux, perm,
                        pos_in);
    }
    const unsigned grid = scatter_grid(a.T * a.k, a.aux.G > 0);
    if (a.dtype == MOE_BF16)
        return launch_k(scatter_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.x), a.idx, a.gate, a.T, a.d, a.N, a.k, a.C,
                        a.claim_base, a.pos, a.drop, a.counts, a.offsets, a.row_token, a.row_gate,
                        reinterpret_cast<__nv_bfloat16*>(a.xe), reinterpret_cast<__nv_bfloat16*>(a.zero_out), a.aux,
                        perm, pos_in);
    return launch_k(scatter_kernel<float>, dim3(grid), dim3(256), 0, s, 1, reinterpret_cast<const float*>(a.x), a.idx,
                    a.gate, a.T, a.d, a.N, a.k, a.C, a.claim_base, a.pos, a.drop, a.counts, a.offsets, a.row_token,
                    a.row_gate, reinterpret_cast<float*>(a.xe), reinterpret_cast<float*>(a.zero_out), a.aux, perm,
                    pos_in);
}

int ntlb_grid_blocks(int64_t T, int sms) {
    const int64_t want = (T + 255) / 256;
    int64_t g = want < sms ? want : sms;
    if (g > kNtlbMaxBlocks) g = kNtlbMaxBlocks;
    return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_dispatch_ntlb(const NtlbArgs& a, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    int sms = 0;
    cudaError_t err = device_sm_count(&sms);
    if (err != cudaSuccess) return err;
    // co-residency: the cooperative launch fails rather than run a grid that does not fit
    const int G = ntlb_grid_blocks(a.T, sms);
    NtlbGrid g{};
    g.probs = a.probs;
    g.T = a.T;
    g.N = a.N;
    g.C = a.C;
    g.TB = (a.T + G - 1) / G;
    g.expert = a.expert;
    g.gate = a.gate;
    g.pos = a.pos;
    g.counts = a.counts;
    g.kept = a.kept;
    g.offsets = a.offsets;
    g.ch = a.ch;
    g.last = a.last;
    g.first = a.first;
    g.placed = a.placed;
    g.lp = a.lp;
    g.agg = a.grid_agg;
    g.unplaced = a.grid_unplaced;
    g.bar = a.grid_bar;
    g.status = &a.hdr->status;
    g.limit_ns = kWaitLimitNs;
    if ((err = cudaMemsetAsync(a.grid_bar, 0, sizeof(uint32_t), s)) != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(kScanThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((err = cudaLaunchKernelEx(&cfg, ntlb_grid_kernel, g)) != cudaSuccess) return err;
    // the gather, from the final experts and claim numbers (rank 0, no claim base)
    const int32_t* none = nullptr;
    const int N = a.N;
    if (a.xe == nullptr && a.zero_out == nullptr) {   // row map only
        const unsigned g2 = (unsigned)((a.T + 255) / 256) + (a.aux.G > 0 ? 1u : 0u);
        return launch_k(rowmap_kernel, dim3(g2), dim3(256), 0, s, 1, static_cast<const int32_t*>(a.expert),
                        static_cast<const float*>(a.gate), a.T, N, 1, a.C, none, a.pos, a.drop,
                        static_cast<const int32_t*>(a.counts), static_cast<const int32_t*>(a.offsets), a.row_token,
                        a.row_gate, a.aux, none, none);
    }
    const unsigned grid = scatter_grid(a.T, a.aux.G > 0);
    if (a.dtype == MOE_BF16)
        return launch_k(scatter_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1,
                        reinterpret_cast<const __nv_bfloat16*>(a.x), static_cast<const int32_t*>(a.expert),
                        static_cast<const float*>(a.gate), a.T, a.d, N, 1, a.C, none, a.pos, a.drop,
                        static_cast<const int32_t*>(a.counts), static_cast<const int32_t*>(a.offsets), a.row_token,
                        a.row_gate, reinterpret_cast<__nv_bfloat16*>(a.xe),
                        reinterpret_cast<__nv_bfloat16*>(a.zero_out), a.aux, none, none);
    return launch_k(scatter_kernel<float>, dim3(grid), dim3(256), 0, s, 1, reinterpret_cast<const float*>(a.x),
                    static_cast<const int32_t*>(a.expert), static_cast<const float*>(a.gate), a.T, a.d, N, 1, a.C,
                    none, a.pos, a.drop, static_cast<const int32_t*>(a.counts),
                    static_cast<const int32_t*>(a.offsets), a.row_token, a.row_gate, reinterpret_cast<float*>(a.xe),
                    reinterpret_cast<float*>(a.zero_out), a.aux, none, none);
}

cudaError_t launch_counts(const int32_t* idx, int64_t T, int N, int k, int32_t* counts, cudaStream_t s) {
    cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)k * N, s);
    if (err != cudaSuccess || T == 0) return err;
    const int64_t n = T * k;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 1024) blocks = 1024;
    count_kernel<<<blocks, 256, 0, s>>>(idx, T, N, k, counts);
    return cudaGetLastError();
}

cudaError_t launch_claim_base(const int32_t* all, int S, int shard, int k, int N, int32_t* base, cudaStream_t s) {
    claim_base_kernel<<<1, 128, 0, s>>>(all, S, shard, k, N, base);
    return cudaGetLastError();
}

cudaError_t launch_aux_shards(int S, int N, const int64_t* tokens, const double* f_all, const double* P_all,
                              float alpha, double* f, double* P, double* aux, cudaStream_t s) {
    aux_shards_kernel<<<1, 128, 0, s>>>(S, N, tokens, f_all, P_all, alpha, f, P, aux);
    return cudaGetLastError();
}

cudaError_t launch_lookback_timeout_probe(uint32_t* state, WsHeader* hdr, long long limit_ns,
                                          cudaStream_t s) {
    cudaError_t err = cudaMemsetAsync(state, 0, 8 * sizeof(uint32_t), s);
    if (err != cudaSuccess) return err;
    lookback_probe_kernel<<<1, 32, 0, s>>>(state, hdr, limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
