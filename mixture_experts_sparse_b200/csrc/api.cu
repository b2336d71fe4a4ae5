// C-ABI front end of libmoe_b200: argument validation, workspace layout and
// the launch sequence of each entry point (declared and documented in
// include/moe.h).  No entry point allocates, frees or synchronises, except
// moe_read_device_status, which synchronises its stream.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace moe {

cudaError_t once_per_device(const void* key, cudaError_t (*set)(const void*)) {
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, cudaError_t> done;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find({dev, key});
    if (it != done.end()) return it->second;
    err = set(key);
    done[{dev, key}] = err;
    return err;
}

bool pdl_enabled() {
    static const bool on = [] {
        const char* v = getenv("MOE_B200_PDL");
        return !(v && strcmp(v, "0") == 0);
    }();
    return on;
}

cudaError_t device_sm_count(int* sms) {
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        err = cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
    }
    *sms = cache[dev];
    return cudaSuccess;
}

namespace {

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
    size_t hdr, part_cnt, part_psum, part_z, w_split, scan_state;
    size_t idx, gate, pos, drop, counts, kept, offsets, f, P, aux;
    size_t row_token, row_gate, xe, h, ye;
    size_t prio_hist, prio_cursor, prio_list, prio_perm, prio_idx, prio_pos, prio_range;   // batch priority only
    size_t ntlb_probs, ntlb_ch, ntlb_last, ntlb_first, ntlb_placed, ntlb_lp;               // re-routing only
    size_t ntlb_agg, ntlb_unplaced, ntlb_bar;
    size_t bwd_part_dw, bwd_part_db;   // router backward partials
    size_t rb_adx, rb_adw, rb_bdx, rb_offs, rb_part;   // router backward on the tensor cores (bf16)
    size_t total;
    int64_t rows;   // min(k T, N C): compact rows the buffers hold
};

int64_t compact_rows(const moe_config& c) {
    int64_t a = (int64_t)c.top_k * c.T;
    int64_t b = (int64_t)c.n_experts * c.capacity;
    return a < b ? a : b;
}

Layout layout_of(const moe_config& c) {
    Layout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += round_up(bytes > 0 ? bytes : 1, 256);
        return o;
    };
    const size_t T = (size_t)c.T, k = (size_t)c.top_k, N = (size_t)c.n_experts;
    const size_t esz = c.dtype == MOE_BF16 ? 2 : 4;
    L.rows = compact_rows(c);
    const size_t R = (size_t)(L.rows > 0 ? L.rows : 1);
    L.hdr = take(sizeof(WsHeader));
    const size_t nbr = (size_t)router_partial_rows(c.T, c.n_experts);
    L.part_cnt = take(4 * nbr * N);
    L.part_psum = take(4 * nbr * N);
    L.part_z = take(8 * nbr);
    L.w_split = take(c.dtype == MOE_BF16 ? 2 * 3 * (size_t)router_tc_padded_experts(c.n_experts) * c.d_model : 0);
    const size_t nbs = (size_t)scan_blocks(c.T);
    L.scan_state = take(4 * (nbs * k * N > 8 ? nbs * k * N : 8));
    L.idx = take(4 * T * k);
    L.gate = take(4 * T * k);
    L.pos = take(4 * T * k);
    L.drop = take(T * k);
    L.counts = take(4 * k * N);
    L.kept = take(4 * N);
    L.offsets = take(4 * (N + 1));
    L.f = take(8 * N);
    L.P = take(8 * N);
    L.aux = take(8);
    L.row_token = take(4 * R);
    L.row_gate = take(4 * R);
    L.xe = take(esz * R * (size_t)c.d_model);
    L.h = take(esz * R * (size_t)c.d_ff);
    L.ye = take(esz * R * (size_t)c.d_model);
    const size_t nch = (size_t)router_bwd_chunks(c.T);
    L.bwd_part_dw = take(4 * nch * N * (size_t)c.d_model);
    L.bwd_part_db = take(4 * nch * N);
    if (c.dtype == MOE_BF16) {
        const size_t np16 = (size_t)router_bwd_np16(c.n_experts), nct = (size_t)router_bwd_tc_chunks(c.T);
        L.rb_adx = take(2 * T * 6 * np16);
        L.rb_adw = take(2 * T * 3 * np16);
        L.rb_bdx = take(2 * 6 * np16 * (size_t)c.d_model);
        L.rb_offs = take(4 * (nct + 3));
        L.rb_part = take(4 * nct * 3 * np16 * (size_t)c.d_model);
    }
    if (c.priority == MOE_ORDER_PRIORITY) {   // batch-priority claim order scratch
        L.prio_hist = take(4 * (size_t)(kPrioBuckets + 1));
        L.prio_cursor = take(4 * (size_t)kPrioBuckets);
        L.prio_list = take(4 * T);
        L.prio_perm = take(4 * T);
        L.prio_idx = take(4 * T * k);
        L.prio_pos = take(4 * T * k);
        L.prio_range = take(8);
    }
    if (c.priority == MOE_ORDER_NTLB) {   // No-Token-Left-Behind scratch
        L.ntlb_probs = take(4 * T * N);
        L.ntlb_ch = take(4 * T);
        L.ntlb_last = take(4 * T);
        L.ntlb_first = take(4 * T);
        L.ntlb_placed = take(4 * T);
        L.ntlb_lp = take(4 * T);
        L.ntlb_agg = take(4 * 2 * (size_t)kNtlbMaxBlocks * N);
        L.ntlb_unplaced = take(4 * 2 * (size_t)kNtlbMaxBlocks);
        L.ntlb_bar = take(4);
    }
    L.total = off;
    return L;
}

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t validate(const moe_config* c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->T < 0 || c->d_model < 1 || c->d_ff < 1 || c->n_experts < 1 || c->top_k < 1 || c->capacity < 0)
        return MOE_ERR_INVALID_ARG;
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (c->act != MOE_RELU && c->act != MOE_SWIGLU) return MOE_ERR_INVALID_ARG;
    if (c->top_k > c->n_experts) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(c->alpha)) return MOE_ERR_INVALID_ARG;
    if (c->priority != MOE_ORDER_TOKEN && c->priority != MOE_ORDER_PRIORITY && c->priority != MOE_ORDER_NTLB)
        return MOE_ERR_INVALID_ARG;
    if (c->T >= (1 << 28) || c->n_experts > 128 || c->top_k > 2) return MOE_ERR_UNSUPPORTED;
    if (c->priority == MOE_ORDER_NTLB && c->top_k != 1) return MOE_ERR_UNSUPPORTED;   // re-routing is top-1
    if (c->dtype == MOE_BF16 && (c->d_model % 16 != 0 || c->d_ff % 16 != 0)) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)c->d_model * c->d_ff >= ((int64_t)1 << 40)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

int32_t validate_config(const moe_config* c) { return validate(c); }

namespace {

int32_t check_ws(const moe_config* c, void* ws, size_t ws_bytes) {
    if (!ws || !aligned(ws)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < layout_of(*c).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

// required pointer: non-null and 16-byte aligned; optional: null or aligned
bool req(const void* p) { return p != nullptr && aligned(p); }
bool opt(const void* p) { return p == nullptr || aligned(p); }

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_capacity(int64_t T, int32_t n_experts, int32_t top_k, double cf) {
    if (T < 0 || n_experts < 1 || top_k < 1 || !(cf >= 0.0) || std::isinf(cf)) return -1;
    if (T == 0 || cf == 0.0) return 0;
    // cf = m * 2^ex exactly, m an integer below 2^53
    int ex = 0;
    double fr = std::frexp(cf, &ex);
    long long m = (long long)std::ldexp(fr, 53);
    ex -= 53;
    while ((m & 1) == 0 && ex < 0) {
        m >>= 1;
        ++ex;
    }
    unsigned __int128 num = (unsigned __int128)top_k * (unsigned __int128)T * (unsigned __int128)m;
    unsigned __int128 den = (unsigned __int128)n_experts;
    if (ex >= 0) {
        if (ex > 60) return -1;
        num <<= ex;
    } else {
        if (-ex > 100) return 0;
        den <<= -ex;
    }
    unsigned __int128 q = num / den;
    if (q > (unsigned __int128)2147483647) return -1;
    return (int32_t)q;
}

size_t moe_workspace_bytes(const moe_config* cfg) {
    if (validate(cfg) != MOE_OK) return 0;
    return layout_of(*cfg).total;
}

int32_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || !aligned(ws) || ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream));
}

const char* moe_status_string(int32_t status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MOE_ERR_CUDA: return "CUDA call failed";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

// The router; with defer (tensor-core router only) its CTAs leave f, P and aux
// to a later aux_reduce_block over their partials.
static int32_t route_impl(const moe_config* cfg, const void* x, const float* w_r, const float* b_r, int32_t* idx,
                          float* gate, float* probs, double* f, double* P, double* aux, void* ws, size_t ws_bytes,
                          void* stream, bool defer, double* z = nullptr) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!req(w_r) || !opt(b_r) || !opt(probs) || !opt(f) || !opt(P) || !opt(aux)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(x) || !req(idx) || !req(gate))) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    const Layout L = layout_of(*cfg);
    RouterArgs a{};
    a.x = x;
    a.dtype = cfg->dtype;
    a.w_r = w_r;
    a.b_r = b_r;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.N = cfg->n_experts;
    a.k = cfg->top_k;
    a.idx = idx;
    a.gate = gate;
    a.probs = probs;
    a.part_cnt = at<int32_t>(ws, L.part_cnt);
    a.part_psum = at<float>(ws, L.part_psum);
    a.part_z = at<double>(ws, L.part_z);
    a.z = z;
    a.f = f;
    a.P = P;
    a.aux = aux;
    a.alpha = cfg->alpha;
    a.w_split = at<void>(ws, L.w_split);
    a.status = &at<WsHeader>(ws, L.hdr)->status;
    a.ticket = &at<WsHeader>(ws, L.hdr)->route_ticket;
    a.defer_aux = defer;
    return cuda_status(launch_router(a, (cudaStream_t)stream));
}

int32_t moe_route(const moe_config* cfg, const void* x, const float* w_r, const float* b_r, int32_t* idx,
                  float* gate, float* probs, double* f, double* P, double* aux, void* ws, size_t ws_bytes,
                  void* stream) {
    return route_impl(cfg, x, w_r, b_r, idx, gate, probs, f, P, aux, ws, ws_bytes, stream, false);
}

int32_t moe_route_z(const moe_config* cfg, const void* x, const float* w_r, const float* b_r, int32_t* idx,
                    float* gate, float* probs, double* f, double* P, double* aux, double* z_loss, void* ws,
                    size_t ws_bytes, void* stream) {
    if (!opt(z_loss)) return MOE_ERR_INVALID_ARG;
    return route_impl(cfg, x, w_r, b_r, idx, gate, probs, f, P, aux, ws, ws_bytes, stream, false, z_loss);
}

static int32_t dispatch_impl(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate,
                             int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept, int32_t* offsets,
                             int32_t* row_token, float* row_gate, void* xe, void* zero_out, void* ws,
                             cudaStream_t s, const int32_t* claim_base = nullptr, const AuxArgs* aux = nullptr) {
    const Layout L = layout_of(*cfg);
    if (cfg->T == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->top_k * cfg->n_experts, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(kept, 0, sizeof(int32_t) * cfg->n_experts, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (cfg->n_experts + 1), s);
        return cuda_status(e);
    }
    DispatchArgs a{};
    a.x = x;
    a.dtype = cfg->dtype;
    a.idx = idx;
    a.gate = gate;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.N = cfg->n_experts;
    a.k = cfg->top_k;
    a.C = cfg->capacity;
    a.pos = pos;
    a.drop = drop;
    a.counts = counts;
    a.kept = kept;
    a.offsets = offsets;
    a.row_token = row_token;
    a.row_gate = row_gate;
    a.xe = xe;
    a.zero_out = zero_out;
    a.scan_state = at<uint32_t>(ws, L.scan_state);
    a.hdr = at<WsHeader>(ws, L.hdr);
    a.claim_base = claim_base;
    if (aux) a.aux = *aux;
    if (cfg->priority == MOE_ORDER_PRIORITY) {
        a.prio.hist = at<int32_t>(ws, L.prio_hist);
        a.prio.cursor = at<int32_t>(ws, L.prio_cursor);
        a.prio.list = at<int32_t>(ws, L.prio_list);
        a.prio.perm = at<int32_t>(ws, L.prio_perm);
        a.prio.idx_sorted = at<int32_t>(ws, L.prio_idx);
        a.prio.pos_sorted = at<int32_t>(ws, L.prio_pos);
        a.prio.range = at<uint32_t>(ws, L.prio_range);
    }
    return cuda_status(launch_dispatch(a, s));
}

// No-Token-Left-Behind dispatch from the router probabilities (top-1).
static int32_t ntlb_impl(const moe_config* cfg, const void* x, const float* probs, int32_t* expert, float* gate,
                         int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept, int32_t* offsets,
                         int32_t* row_token, float* row_gate, void* xe, void* zero_out, void* ws, cudaStream_t s,
                         const AuxArgs* aux = nullptr) {
    const Layout L = layout_of(*cfg);
    if (cfg->T == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(kept, 0, sizeof(int32_t) * cfg->n_experts, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (cfg->n_experts + 1), s);
        return cuda_status(e);
    }
    NtlbArgs a{};
    a.x = x;
    a.dtype = cfg->dtype;
    a.probs = probs;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.N = cfg->n_experts;
    a.C = cfg->capacity;
    a.expert = expert;
    a.gate = gate;
    a.pos = pos;
    a.drop = drop;
    a.counts = counts;
    a.kept = kept;
    a.offsets = offsets;
    a.row_token = row_token;
    a.row_gate = row_gate;
    a.xe = xe;
    a.zero_out = zero_out;
    a.ch = at<int32_t>(ws, L.ntlb_ch);
    a.last = at<int32_t>(ws, L.ntlb_last);
    a.first = at<int32_t>(ws, L.ntlb_first);
    a.placed = at<int32_t>(ws, L.ntlb_placed);
    a.lp = at<int32_t>(ws, L.ntlb_lp);
    a.grid_agg = at<int32_t>(ws, L.ntlb_agg);
    a.grid_unplaced = at<int32_t>(ws, L.ntlb_unplaced);
    a.grid_bar = at<uint32_t>(ws, L.ntlb_bar);
    a.hdr = at<WsHeader>(ws, L.hdr);
    if (aux) a.aux = *aux;
    return cuda_status(launch_dispatch_ntlb(a, s));
}

int32_t moe_dispatch_ntlb(const moe_config* cfg, const void* x, const float* probs, int32_t* expert, float* gate,
                          int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept, int32_t* offsets,
                          int32_t* row_token, float* row_gate, void* xe, void* ws, size_t ws_bytes, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->priority != MOE_ORDER_NTLB) return MOE_ERR_INVALID_ARG;
    if (!req(counts) || !req(kept) || !req(offsets) || !opt(xe) || !opt(x)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(probs) || !req(expert) || !req(gate) || !req(pos) || !req(drop) || !req(row_token) ||
                       !req(row_gate)))
        return MOE_ERR_INVALID_ARG;
    if (xe && cfg->T > 0 && !req(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    return ntlb_impl(cfg, x, probs, expert, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, nullptr,
                     ws, (cudaStream_t)stream);
}

int32_t moe_gate_grad(const moe_config* cfg, const void* dout, const void* ye, const int32_t* idx,
                      const int32_t* pos, const uint8_t* drop, const int32_t* offsets, float* dgate, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->T > 0 && (!req(dout) || !req(idx) || !req(pos) || !req(drop) || !req(offsets) || !req(dgate)))
        return MOE_ERR_INVALID_ARG;
    if (!opt(ye)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && compact_rows(*cfg) > 0 && !ye) return MOE_ERR_INVALID_ARG;
    GateGradArgs a{};
    a.dtype = cfg->dtype;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.k = cfg->top_k;
    a.dout = dout;
    a.ye = ye;
    a.idx = idx;
    a.pos = pos;
    a.drop = drop;
    a.offsets = offsets;
    a.dgate = dgate;
    return cuda_status(launch_gate_grad(a, (cudaStream_t)stream));
}

int32_t moe_router_backward(const moe_config* cfg, const void* x, const float* w_r, const float* probs,
                            const int32_t* idx, const float* gate, const double* f, const float* dgate, float* dh,
                            float* dw_r, float* db_r, float* dx, void* ws, size_t ws_bytes, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!req(w_r) || !req(f) || !opt(dw_r) || !opt(db_r) || !opt(dx)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(x) || !req(probs) || !req(idx) || !req(gate) || !req(dgate) || !req(dh)))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    const Layout L = layout_of(*cfg);
    RouterBwdArgs a{};
    a.x = x;
    a.dtype = cfg->dtype;
    a.w_r = w_r;
    a.probs = probs;
    a.idx = idx;
    a.gate = gate;
    a.f = f;
    a.dgate = dgate;
    a.alpha = cfg->alpha;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.N = cfg->n_experts;
    a.k = cfg->top_k;
    a.dh = dh;
    a.dw = dw_r;
    a.db = db_r;
    a.dx = dx;
    a.part_dw = at<float>(ws, L.bwd_part_dw);
    a.part_db = at<float>(ws, L.bwd_part_db);
    if (cfg->dtype == MOE_BF16) {
        a.tc_adx = at<void>(ws, L.rb_adx);
        a.tc_adw = at<void>(ws, L.rb_adw);
        a.tc_bdx = at<void>(ws, L.rb_bdx);
        a.tc_offs = at<int32_t>(ws, L.rb_offs);
        a.tc_part = at<float>(ws, L.rb_part);
    }
    a.status = &at<WsHeader>(ws, L.hdr)->status;
    return cuda_status(launch_router_backward(a, (cudaStream_t)stream));
}

int32_t moe_dispatch(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate, int32_t* pos,
                     uint8_t* drop, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_token,
                     float* row_gate, void* xe, void* ws, size_t ws_bytes, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!req(counts) || !req(kept) || !req(offsets) || !opt(xe) || !opt(x)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(idx) || !req(gate) || !req(pos) || !req(drop) || !req(row_token) || !req(row_gate)))
        return MOE_ERR_INVALID_ARG;
    if (xe && cfg->T > 0 && !req(x)) return MOE_ERR_INVALID_ARG;
    if (cfg->priority == MOE_ORDER_NTLB) return MOE_ERR_UNSUPPORTED;   // needs the probabilities: moe_dispatch_ntlb
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    return dispatch_impl(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, nullptr, ws,
                         (cudaStream_t)stream);
}

int32_t moe_dispatch_shard(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate,
                           const int32_t* claim_base, int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept,
                           int32_t* offsets, int32_t* row_token, float* row_gate, void* xe, void* ws,
                           size_t ws_bytes, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->priority != MOE_ORDER_TOKEN) return MOE_ERR_UNSUPPORTED;   // needs every shard's scores
    if (!req(claim_base) || !req(counts) || !req(kept) || !req(offsets) || !opt(xe) || !opt(x))
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(idx) || !req(gate) || !req(pos) || !req(drop) || !req(row_token) || !req(row_gate)))
        return MOE_ERR_INVALID_ARG;
    if (xe && cfg->T > 0 && !req(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    return dispatch_impl(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, nullptr, ws,
                         (cudaStream_t)stream, claim_base);
}

int32_t moe_expert_counts(const moe_config* cfg, const int32_t* idx, int32_t* counts, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!req(counts) || (cfg->T > 0 && !req(idx))) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_counts(idx, cfg->T, cfg->n_experts, cfg->top_k, counts, (cudaStream_t)stream));
}

int32_t moe_claim_base(const int32_t* shard_counts, int32_t n_shards, int32_t shard, int32_t top_k,
                       int32_t n_experts, int32_t* claim_base, void* stream) {
    if (n_shards < 1 || shard < 0 || shard >= n_shards || top_k < 1 || n_experts < 1) return MOE_ERR_INVALID_ARG;
    if (top_k > 2 || n_experts > 128) return MOE_ERR_UNSUPPORTED;
    if (!req(shard_counts) || !req(claim_base)) return MOE_ERR_INVALID_ARG;
    return cuda_status(
        launch_claim_base(shard_counts, n_shards, shard, top_k, n_experts, claim_base, (cudaStream_t)stream));
}

int32_t moe_aux_shards(int32_t n_shards, int32_t n_experts, const int64_t* shard_tokens, const double* f_all,
                       const double* P_all, float alpha, double* f, double* P, double* aux, void* stream) {
    if (n_shards < 1 || n_experts < 1 || !std::isfinite(alpha)) return MOE_ERR_INVALID_ARG;
    if (n_experts > 128) return MOE_ERR_UNSUPPORTED;
    if (!req(shard_tokens) || !req(f_all) || !req(P_all) || !opt(f) || !opt(P) || !opt(aux))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(
        launch_aux_shards(n_shards, n_experts, shard_tokens, f_all, P_all, alpha, f, P, aux, (cudaStream_t)stream));
}

static int32_t ffn_impl(const moe_config* cfg, const void* xe, const int32_t* offsets, const void* w1,
                        const void* b1, const void* w3, const void* b3, const void* w2, const void* b2, void* ye,
                        void* scatter_out, const int32_t* row_token, const float* row_gate, void* ws,
                        cudaStream_t s, void* const* mid_event = nullptr) {
    const Layout L = layout_of(*cfg);
    if (L.rows <= 0) {   // nothing can be kept
        if (mid_event && *mid_event) return cuda_status(cudaEventRecord((cudaEvent_t)*mid_event, s));
        return MOE_OK;
    }
    FfnArgs a{};
    a.dtype = cfg->dtype;
    a.act = cfg->act;
    a.N = cfg->n_experts;
    a.d = cfg->d_model;
    a.d_ff = cfg->d_ff;
    a.C = (int)(L.rows < cfg->capacity ? L.rows : cfg->capacity);
    a.R_cap = L.rows;
    a.xe = xe;
    a.offsets = offsets;
    a.w1 = w1;
    a.b1 = b1;
    a.w3 = w3;
    a.b3 = b3;
    a.w2 = w2;
    a.b2 = b2;
    a.h = at<void>(ws, L.h);
    a.ye = ye;
    a.scatter_out = scatter_out;
    a.row_token = row_token;
    a.row_gate = row_gate;
    a.hdr = at<WsHeader>(ws, L.hdr);
    a.mid_event = mid_event ? *mid_event : nullptr;
    return cuda_status(launch_expert_ffn(a, s));
}

int32_t moe_expert_ffn(const moe_config* cfg, const void* xe, const int32_t* offsets, const void* w1, const void* b1,
                       const void* w3, const void* b3, const void* w2, const void* b2, void* ye, void* ws,
                       size_t ws_bytes, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!req(xe) || !req(offsets) || !req(w1) || !req(w2) || !req(ye) || !opt(b1) || !opt(b2) || !opt(b3))
        return MOE_ERR_INVALID_ARG;
    if (cfg->act == MOE_SWIGLU ? !req(w3) : !opt(w3)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    return ffn_impl(cfg, xe, offsets, w1, b1, w3, b3, w2, b2, ye, nullptr, nullptr, nullptr, ws,
                    (cudaStream_t)stream);
}

static int32_t combine_impl(const moe_config* cfg, const void* ye, const int32_t* idx, const int32_t* pos,
                            const uint8_t* drop, const float* gate, const int32_t* offsets,
                            const int32_t* claim_base, const int32_t* counts, void* out, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->T > 0 && (!req(idx) || !req(pos) || !req(drop) || !req(gate) || !req(offsets) || !req(out)))
        return MOE_ERR_INVALID_ARG;
    if (!opt(ye) || !opt(claim_base) || !opt(counts)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && compact_rows(*cfg) > 0 && !ye) return MOE_ERR_INVALID_ARG;
    CombineArgs a{};
    a.dtype = cfg->dtype;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.k = cfg->top_k;
    a.ye = ye;
    a.idx = idx;
    a.pos = pos;
    a.drop = drop;
    a.gate = gate;
    a.offsets = offsets;
    a.out = out;
    a.claim_base = claim_base;
    a.counts = counts;
    a.C = (int)cfg->capacity;
    a.N = (int)cfg->n_experts;
    return cuda_status(launch_combine(a, (cudaStream_t)stream));
}

int32_t moe_combine(const moe_config* cfg, const void* ye, const int32_t* idx, const int32_t* pos,
                    const uint8_t* drop, const float* gate, const int32_t* offsets, void* out, void* stream) {
    return combine_impl(cfg, ye, idx, pos, drop, gate, offsets, nullptr, nullptr, out, stream);
}

int32_t moe_combine_shard(const moe_config* cfg, const void* ye, const int32_t* idx, const int32_t* pos,
                          const uint8_t* drop, const float* gate, const int32_t* offsets,
                          const int32_t* claim_base, const int32_t* counts, void* out, void* stream) {
    if (!claim_base || !counts) return MOE_ERR_INVALID_ARG;
    return combine_impl(cfg, ye, idx, pos, drop, gate, offsets, claim_base, counts, out, stream);
}

static int32_t forward_impl(const moe_config* cfg, const void* x, const float* w_r, const float* b_r,
                            const void* w1, const void* b1, const void* w3, const void* b3, const void* w2,
                            const void* b2, void* out, int32_t* idx, float* gate, int32_t* pos, uint8_t* drop,
                            int32_t* counts, int32_t* kept, int32_t* offsets, double* f, double* P, double* aux,
                            void* ws, size_t ws_bytes, cudaStream_t s, void* const* events) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!req(w_r) || !req(w1) || !req(w2) || !opt(b_r) || !opt(b1) || !opt(b2) || !opt(b3)) return MOE_ERR_INVALID_ARG;
    if (cfg->act == MOE_SWIGLU ? !req(w3) : !opt(w3)) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(x) || !req(out))) return MOE_ERR_INVALID_ARG;
    if (!opt(idx) || !opt(gate) || !opt(pos) || !opt(drop) || !opt(counts) || !opt(kept) || !opt(offsets) || !opt(f) ||
        !opt(P) || !opt(aux))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    const Layout L = layout_of(*cfg);
    auto mark = [&](int i) -> bool {
        if (!events || !events[i]) return true;
        return cudaEventRecord((cudaEvent_t)events[i], s) == cudaSuccess;
    };
    if (!idx) idx = at<int32_t>(ws, L.idx);
    if (!gate) gate = at<float>(ws, L.gate);
    if (!pos) pos = at<int32_t>(ws, L.pos);
    if (!drop) drop = at<uint8_t>(ws, L.drop);
    if (!counts) counts = at<int32_t>(ws, L.counts);
    if (!kept) kept = at<int32_t>(ws, L.kept);
    if (!offsets) offsets = at<int32_t>(ws, L.offsets);
    if (!f) f = at<double>(ws, L.f);
    if (!P) P = at<double>(ws, L.P);
    if (!aux) aux = at<double>(ws, L.aux);
    int32_t* row_token = at<int32_t>(ws, L.row_token);
    float* row_gate = at<float>(ws, L.row_gate);
    void* xe = at<void>(ws, L.xe);
    void* ye = at<void>(ws, L.ye);

    if (!mark(0)) return MOE_ERR_CUDA;
    // bf16: the router's CTAs leave the load-balancing loss to one extra block
    // of the gather, which runs beside the HBM-bound row copies
    const bool defer = cfg->dtype == MOE_BF16 && cfg->T > 0;
    AuxArgs aa{};
    if (defer && (f || P || aux)) {
        int sms = 0;
        if (device_sm_count(&sms) != cudaSuccess) return MOE_ERR_CUDA;
        aa = AuxArgs{at<int32_t>(ws, L.part_cnt), at<float>(ws, L.part_psum), router_tc_grid(cfg->T, sms),
                     (int)cfg->n_experts, cfg->T, cfg->alpha, f, P, aux, nullptr, nullptr};
    }
    // re-routing needs every token's router probabilities
    const bool ntlb = cfg->priority == MOE_ORDER_NTLB;
    float* probs_ws = ntlb ? at<float>(ws, L.ntlb_probs) : nullptr;
    st = route_impl(cfg, x, w_r, b_r, idx, gate, probs_ws, f, P, aux, ws, ws_bytes, s, defer);
    if (st != MOE_OK) return st;
    if (!mark(1)) return MOE_ERR_CUDA;
    // top-1 bf16: the second GEMM scatters gate * E(x) into out; dispatch zeroes
    // the rows of dropped tokens.  Otherwise expert outputs go through the combine.
    const bool fused = cfg->dtype == MOE_BF16 && cfg->top_k == 1;
    // re-routing overwrites idx and gate with the expert each token finally uses and its probability
    st = ntlb ? ntlb_impl(cfg, x, probs_ws, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe,
                          fused ? out : nullptr, ws, s, aa.G > 0 ? &aa : nullptr)
              : dispatch_impl(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe,
                              fused ? out : nullptr, ws, s, nullptr, aa.G > 0 ? &aa : nullptr);
    if (st != MOE_OK) return st;
    if (!mark(2)) return MOE_ERR_CUDA;
    st = ffn_impl(cfg, xe, offsets, w1, b1, w3, b3, w2, b2, ye, fused ? out : nullptr, row_token, row_gate, ws, s,
                  events ? events + 3 : nullptr);
    if (st != MOE_OK) return st;
    if (!mark(4)) return MOE_ERR_CUDA;
    if (!fused) {
        CombineArgs a{};
        a.dtype = cfg->dtype;
        a.T = cfg->T;
        a.d = cfg->d_model;
        a.k = cfg->top_k;
        a.ye = ye;
        a.idx = idx;
        a.pos = pos;
        a.drop = drop;
        a.gate = gate;
        a.offsets = offsets;
        a.out = out;
        st = cuda_status(launch_combine(a, s));
        if (st != MOE_OK) return st;
    }
    if (!mark(5)) return MOE_ERR_CUDA;
    return MOE_OK;
}

int32_t moe_forward(const moe_config* cfg, const void* x, const float* w_r, const float* b_r, const void* w1,
                    const void* b1, const void* w3, const void* b3, const void* w2, const void* b2, void* out,
                    int32_t* idx, float* gate, int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept,
                    int32_t* offsets, double* f, double* P, double* aux, void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(cfg, x, w_r, b_r, w1, b1, w3, b3, w2, b2, out, idx, gate, pos, drop, counts, kept, offsets,
                        f, P, aux, ws, ws_bytes, (cudaStream_t)stream, nullptr);
}

int32_t moe_forward_events(const moe_config* cfg, const void* x, const float* w_r, const float* b_r,
                           const void* w1, const void* b1, const void* w3, const void* b3, const void* w2,
                           const void* b2, void* out, int32_t* idx, float* gate, int32_t* pos, uint8_t* drop,
                           int32_t* counts, int32_t* kept, int32_t* offsets, double* f, double* P, double* aux,
                           void* ws, size_t ws_bytes, void* stream, void* const* events) {
    return forward_impl(cfg, x, w_r, b_r, w1, b1, w3, b3, w2, b2, out, idx, gate, pos, drop, counts, kept, offsets,
                        f, P, aux, ws, ws_bytes, (cudaStream_t)stream, events);
}

// ---- expert FFN backward ---------------------------------------------------

struct BwdLayout {
    size_t hdr, h, pre, dy, du, dxe, total;
    int64_t rows;
};

static BwdLayout bwd_layout(const moe_config& c) {
    BwdLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += round_up(bytes > 0 ? bytes : 1, 256);
        return o;
    };
    L.rows = compact_rows(c);
    const size_t R = (size_t)(L.rows > 0 ? L.rows : 1), d = (size_t)c.d_model, dff = (size_t)c.d_ff;
    const bool sw = c.act == MOE_SWIGLU;
    L.hdr = take(sizeof(WsHeader));
    L.h = take(2 * R * dff);
    L.pre = take(sw ? 2 * R * 2 * dff : 0);
    L.dy = take(2 * R * d);
    L.du = take(2 * R * (sw ? 2 : 1) * dff);
    L.dxe = take(c.top_k == 2 ? 4 * R * d : 0);
    L.total = off;
    return L;
}

size_t moe_expert_backward_workspace_bytes(const moe_config* cfg) {
    if (validate(cfg) != MOE_OK || cfg->dtype != MOE_BF16) return 0;
    return bwd_layout(*cfg).total;
}

int32_t moe_expert_backward(const moe_config* cfg, const void* xe, const int32_t* offsets, const int32_t* row_token,
                            const float* row_gate, const int32_t* idx, const int32_t* pos, const uint8_t* drop,
                            const void* dout, const void* w1, const void* b1, const void* w3, const void* b3,
                            const void* w2, float* dx, float* dw1, float* db1, float* dw3, float* db3, float* dw2,
                            float* db2, void* ws, size_t ws_bytes, void* stream) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;   // the tensor-core backward is bf16
    // SwiGLU: the dx GEMM reads W1 then W3 along K in 64-row blocks
    if (cfg->act == MOE_SWIGLU && cfg->d_ff % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (!req(offsets) || !req(w1) || !req(w2) || !opt(b1) || !opt(b3) || !opt(dw1) || !opt(db1) || !opt(dw3) ||
        !opt(db3) || !opt(dw2) || !opt(db2) || !opt(dx))
        return MOE_ERR_INVALID_ARG;
    if (cfg->act == MOE_SWIGLU ? !req(w3) : !opt(w3)) return MOE_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(*cfg);
    if (!ws || !aligned(ws) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (cfg->T > 0 && (!req(xe) || !req(row_token) || !req(row_gate) || !req(idx) || !req(pos) || !req(drop) ||
                       !req(dout) || !req(dx)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    // an expert with no rows has zero weight gradients; the kernels write them too
    if (L.rows <= 0 || cfg->T == 0) {
        cudaError_t e = cudaSuccess;
        const size_t N = (size_t)cfg->n_experts, d = (size_t)cfg->d_model, dff = (size_t)cfg->d_ff;
        if (dw1) e = cudaMemsetAsync(dw1, 0, 4 * N * dff * d, s);
        if (e == cudaSuccess && dw3) e = cudaMemsetAsync(dw3, 0, 4 * N * dff * d, s);
        if (e == cudaSuccess && dw2) e = cudaMemsetAsync(dw2, 0, 4 * N * dff * d, s);
        if (e == cudaSuccess && db1) e = cudaMemsetAsync(db1, 0, 4 * N * dff, s);
        if (e == cudaSuccess && db3) e = cudaMemsetAsync(db3, 0, 4 * N * dff, s);
        if (e == cudaSuccess && db2) e = cudaMemsetAsync(db2, 0, 4 * N * d, s);
        if (e == cudaSuccess && dx && cfg->T > 0) e = cudaMemsetAsync(dx, 0, 4 * (size_t)cfg->T * d, s);
        return cuda_status(e);
    }
    BwdArgs a{};
    a.act = cfg->act;
    a.N = cfg->n_experts;
    a.d = cfg->d_model;
    a.d_ff = cfg->d_ff;
    a.k = cfg->top_k;
    a.T = cfg->T;
    a.R_cap = L.rows;
    a.xe = xe;
    a.offsets = offsets;
    a.row_token = row_token;
    a.row_gate = row_gate;
    a.idx = idx;
    a.pos = pos;
    a.drop = drop;
    a.dout = dout;
    a.w1 = w1;
    a.b1 = b1;
    a.w3 = w3;
    a.b3 = b3;
    a.w2 = w2;
    a.dx = dx;
    a.dw1 = dw1;
    a.db1 = db1;
    a.dw3 = dw3;
    a.db3 = db3;
    a.dw2 = dw2;
    a.db2 = db2;
    a.top1_scatter = cfg->top_k == 1;
    a.h = at<void>(ws, L.h);
    a.pre = at<void>(ws, L.pre);
    a.dy = at<void>(ws, L.dy);
    a.du = at<void>(ws, L.du);
    a.dxe = at<float>(ws, L.dxe);
    a.hdr = at<WsHeader>(ws, L.hdr);
    return cuda_status(launch_expert_backward_tc(a, s));
}

// ---- expert parallelism --------------------------------------------------

// The receiving GPU's view of a layer split over n_ranks GPUs: its E = N / G
// experts, and up to min(k T, E C) rows from each of the G sources.
static bool ep_recv_config(const moe_config* cfg, int32_t n_ranks, moe_config* out) {
    if (!cfg || n_ranks < 1 || cfg->n_experts % n_ranks != 0) return false;
    moe_config r = *cfg;
    const int64_t T = (int64_t)cfg->T * n_ranks, C = (int64_t)cfg->capacity * n_ranks;
    if (T >= (int64_t)1 << 28 || C > 2147483647) return false;
    r.T = (int32_t)T;
    r.n_experts = cfg->n_experts / n_ranks;
    r.capacity = (int32_t)C;
    r.top_k = cfg->top_k > r.n_experts ? r.n_experts : cfg->top_k;   // only sizes depend on it here
    *out = r;
    return true;
}

static int32_t ep_check(const moe_config* cfg, int32_t n_ranks, int32_t rank) {
    int32_t st = validate(cfg);
    if (st != MOE_OK) return st;
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks) return MOE_ERR_INVALID_ARG;
    if (cfg->n_experts % n_ranks != 0) return MOE_ERR_UNSUPPORTED;   // whole experts per GPU
    if (cfg->priority != MOE_ORDER_TOKEN) return MOE_ERR_UNSUPPORTED;
    moe_config r;
    if (!ep_recv_config(cfg, n_ranks, &r) || validate(&r) != MOE_OK) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int64_t moe_ep_recv_rows(const moe_config* cfg, int32_t n_ranks) {
    moe_config r;
    if (ep_check(cfg, n_ranks, 0) != MOE_OK || !ep_recv_config(cfg, n_ranks, &r)) return -1;
    return compact_rows(r);
}

size_t moe_ep_workspace_bytes(const moe_config* cfg, int32_t n_ranks) {
    moe_config r;
    if (ep_check(cfg, n_ranks, 0) != MOE_OK || !ep_recv_config(cfg, n_ranks, &r)) return 0;
    return layout_of(r).total;
}

int32_t moe_ep_layout(int32_t n_ranks, int32_t rank, int32_t n_experts, const int32_t* kept_all, int32_t* dst_start,
                      int32_t* recv_offsets, void* stream) {
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks || n_experts < 1) return MOE_ERR_INVALID_ARG;
    if (n_experts > 128 || n_experts % n_ranks != 0) return MOE_ERR_UNSUPPORTED;
    if (!req(kept_all) || !req(dst_start) || !req(recv_offsets)) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_ep_layout(n_ranks, rank, n_experts, kept_all, dst_start, recv_offsets,
                                        (cudaStream_t)stream));
}

int32_t moe_ep_dispatch(const moe_config* cfg, int32_t n_ranks, int32_t rank, const void* x, const int32_t* offsets,
                        const int32_t* row_token, const float* row_gate, const uint8_t* drop,
                        const int32_t* dst_start, void* const* recv_x, int32_t* const* recv_rank,
                        int32_t* const* recv_row, float* const* recv_gate, void* out, void* stream) {
    int32_t st = ep_check(cfg, n_ranks, rank);
    if (st != MOE_OK) return st;
    if (!req(offsets) || !req(dst_start) || !req(recv_x) || !req(recv_rank) || !req(recv_row) || !req(recv_gate) ||
        !opt(out))
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!req(x) || !req(row_token) || !req(row_gate) || !req(drop))) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && cfg->top_k == 1 && !out) return MOE_ERR_INVALID_ARG;   // dropped tokens' rows are zeroed
    EpDispatchArgs a{};
    a.dtype = cfg->dtype;
    a.T = cfg->T;
    a.d = cfg->d_model;
    a.N = cfg->n_experts;
    a.k = cfg->top_k;
    a.G = n_ranks;
    a.rank = rank;
    a.R_cap = compact_rows(*cfg);
    a.x = x;
    a.offsets = offsets;
    a.row_token = row_token;
    a.row_gate = row_gate;
    a.dst_start = dst_start;
    a.drop = drop;
    a.out = cfg->top_k == 1 ? out : nullptr;
    a.recv_x = recv_x;
    a.recv_rank = recv_rank;
    a.recv_row = recv_row;
    a.recv_gate = recv_gate;
    return cuda_status(launch_ep_dispatch(a, (cudaStream_t)stream));
}

int32_t moe_ep_expert_ffn(const moe_config* cfg, int32_t n_ranks, const void* recv_x, const int32_t* recv_offsets,
                          const void* w1, const void* b1, const void* w3, const void* b3, const void* w2,
                          const void* b2, const int32_t* recv_rank, const int32_t* recv_row, const float* recv_gate,
                          void* const* out_ptrs, void* ws, size_t ws_bytes, void* stream) {
    int32_t st = ep_check(cfg, n_ranks, 0);
    if (st != MOE_OK) return st;
    moe_config r;
    ep_recv_config(cfg, n_ranks, &r);
    if (!req(recv_x) || !req(recv_offsets) || !req(w1) || !req(w2) || !opt(b1) || !opt(b2) || !opt(b3) ||
        !req(recv_rank) || !req(recv_row) || !req(out_ptrs) || !opt(recv_gate))
        return MOE_ERR_INVALID_ARG;
    if (cfg->act == MOE_SWIGLU ? !req(w3) : !opt(w3)) return MOE_ERR_INVALID_ARG;
    if (cfg->top_k == 1 && !recv_gate) return MOE_ERR_INVALID_ARG;   // top-1 results leave gated
    if ((st = check_ws(&r, ws, ws_bytes)) != MOE_OK) return st;
    const Layout L = layout_of(r);
    if (L.rows <= 0) return MOE_OK;
    cudaStream_t s = (cudaStream_t)stream;
    // top-1: gate * E(x) into the source's out row of the token; top-2: E(x)
    // into the source's compact row (the source's combine applies the gates)
    const float* g = cfg->top_k == 1 ? recv_gate : nullptr;
    if (cfg->dtype == MOE_BF16) {
        FfnArgs a{};
        a.dtype = r.dtype;
        a.act = r.act;
        a.N = r.n_experts;
        a.d = r.d_model;
        a.d_ff = r.d_ff;
        a.C = (int)(L.rows < r.capacity ? L.rows : r.capacity);
        a.R_cap = L.rows;
        a.xe = recv_x;
        a.offsets = recv_offsets;
        a.w1 = w1;
        a.b1 = b1;
        a.w3 = w3;
        a.b3 = b3;
        a.w2 = w2;
        a.b2 = b2;
        a.h = at<void>(ws, L.h);
        a.ye = at<void>(ws, L.ye);
        a.row_token = recv_row;
        a.row_gate = g;
        a.scatter_ptrs = out_ptrs;
        a.row_rank = recv_rank;
        a.hdr = at<WsHeader>(ws, L.hdr);
        return cuda_status(launch_expert_ffn(a, s));
    }
    // fp32: the FP32-pipe expert FFN into the workspace, then the rows go back
    st = ffn_impl(&r, recv_x, recv_offsets, w1, b1, w3, b3, w2, b2, at<void>(ws, L.ye), nullptr, nullptr, nullptr,
                  ws, s);
    if (st != MOE_OK) return st;
    return cuda_status(launch_ep_return(r.dtype, at<void>(ws, L.ye), recv_offsets, r.n_experts, r.d_model, L.rows,
                                        recv_rank, recv_row, g, out_ptrs, s));
}

int32_t moe_read_device_status(void* ws, void* stream) {
    if (!ws || !aligned(ws)) return MOE_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    int32_t host = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(&host, &hdr->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (host != MOE_OK) {   // a call gave up: clear the status and the per-call counters
        if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return host;
}

int32_t moe_test_lookback_timeout(void* ws, size_t ws_bytes, int64_t limit_ns, void* stream) {
    if (!ws || !aligned(ws) || ws_bytes < sizeof(WsHeader) + 256) return MOE_ERR_WORKSPACE;
    if (limit_ns <= 0 || limit_ns > 10000000000LL) return MOE_ERR_INVALID_ARG;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    uint32_t* state = at<uint32_t>(ws, sizeof(WsHeader));
    return cuda_status(launch_lookback_timeout_probe(state, hdr, (long long)limit_ns, (cudaStream_t)stream));
}

}  // extern "C"
