// moe_dispatch_noalloc: the capacity-limited dispatch with its scratch memory
// held by the library instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: plugin interfaces that
// pass a kernel only its input and output tensors, and serving runtimes that
// reserve all device memory when they start and do not allow cudaMalloc
// afterwards (it synchronises the device and can fail once memory is
// fragmented).  This entry point needs no allocation from them: the look-back
// scratch of the dispatch scan (a status/counter header plus one flag word per
// block and (rank, expert) counter) lives in a file-scope __device__ array of
// fixed size, so every GPU that loads the library holds kNoAllocBytes (about
// 256 KB) until the process exits.
//
// Rules that follow from the shared array:
//   - T may not exceed kNoAllocMaxTokens (262144); larger T returns
//     MOE_ERR_UNSUPPORTED before anything is launched.
//   - The array keeps the previous call's contents; each call clears the part
//     it uses (header and flags) on its stream before the scan runs.
//   - Calls whose work can overlap on the same GPU (different streams, or
//     different host threads on one device) race on the array and must be
//     serialised by the caller.
//   - The device address of the array is looked up once per device, on the
//     first call made with that device current; make that first call before
//     any stream capture begins.  The address is kept for the life of the
//     process, which assumes the device's primary context lives as long (no
//     cudaDeviceReset between calls).
// The kernels launched are those of moe_dispatch.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int64_t kNoAllocMaxTokens = int64_t(1) << 18;
// one look-back word per (scan block, rank, expert) at the largest T, k and N
constexpr size_t kNoAllocFlagWords = (size_t)((kNoAllocMaxTokens + kScanTokens - 1) / kScanTokens) * 2 * 128;
constexpr size_t kNoAllocBytes = sizeof(WsHeader) + kNoAllocFlagWords * sizeof(uint32_t);

}  // namespace
}  // namespace moe

// The scratch itself.  In host code this name is only a host-side stand-in for
// the device object: never pass it to a kernel, use scratch_base() instead.
static __device__ __align__(256) unsigned char g_dispatch_scratch[moe::kNoAllocBytes];

namespace moe {
namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64];

// Device address of g_dispatch_scratch on the current device (looked up once
// per device with cudaGetSymbolAddress).
cudaError_t scratch_base(void** out) {
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool req16(const void* p) { return p != nullptr && aligned16(p); }
bool opt16(const void* p) { return p == nullptr || aligned16(p); }

}  // namespace
}  // namespace moe

extern "C" int32_t moe_dispatch_noalloc(const moe_config* cfg, const void* x, const int32_t* idx, const float* gate,
                                        int32_t* pos, uint8_t* drop, int32_t* counts, int32_t* kept,
                                        int32_t* offsets, int32_t* row_token, float* row_gate, void* xe,
                                        int32_t* status, void* stream) {
    using namespace moe;
    const int32_t st = validate_config(cfg);   // the checks every entry point makes
    if (st != MOE_OK) return st;
    const moe_config& c = *cfg;
    if (c.priority != MOE_ORDER_TOKEN) return MOE_ERR_UNSUPPORTED;   // its scratch has no room for the sort
    if (c.T > kNoAllocMaxTokens ||   // beyond the static scratch
        (size_t)scan_blocks(c.T) * c.top_k * c.n_experts > kNoAllocFlagWords)
        return MOE_ERR_UNSUPPORTED;
    if (!req16(counts) || !req16(kept) || !req16(offsets) || !opt16(xe) || !opt16(x) || !opt16(status))
        return MOE_ERR_INVALID_ARG;
    if (c.T > 0 && (!req16(idx) || !req16(gate) || !req16(pos) || !req16(drop) || !req16(row_token) ||
                    !req16(row_gate)))
        return MOE_ERR_INVALID_ARG;
    if (xe && c.T > 0 && !req16(x)) return MOE_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    void* base = nullptr;
    if (scratch_base(&base) != cudaSuccess) return MOE_ERR_CUDA;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
    if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return MOE_ERR_CUDA;
    cudaError_t err = cudaSuccess;
    if (c.T == 0) {
        err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * c.top_k * c.n_experts, s);
        if (err == cudaSuccess) err = cudaMemsetAsync(kept, 0, sizeof(int32_t) * c.n_experts, s);
        if (err == cudaSuccess) err = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (c.n_experts + 1), s);
    } else {
        DispatchArgs a{};
        a.x = x;
        a.dtype = c.dtype;
        a.idx = idx;
        a.gate = gate;
        a.T = c.T;
        a.d = c.d_model;
        a.N = c.n_experts;
        a.k = c.top_k;
        a.C = c.capacity;
        a.pos = pos;
        a.drop = drop;
        a.counts = counts;
        a.kept = kept;
        a.offsets = offsets;
        a.row_token = row_token;
        a.row_gate = row_gate;
        a.xe = xe;
        a.zero_out = nullptr;
        a.scan_state = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(base) + sizeof(WsHeader));
        a.hdr = hdr;
        err = launch_dispatch(a, s);
    }
    if (err == cudaSuccess && status)   // device-side status of this call (MOE_OK or MOE_ERR_TIMEOUT)
        err = cudaMemcpyAsync(status, &hdr->status, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
