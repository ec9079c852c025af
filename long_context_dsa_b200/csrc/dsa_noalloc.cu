// dsa_noalloc.cu -- idx_score_topk for callers that cannot allocate device
// memory.
//
// Some callers have no way to hand the library a workspace: a plug-in that
// runs inside another runtime whose memory pool owns every device
// allocation (and forbids cudaMalloc, which may also synchronise the whole
// device), or code on a latency-critical path that must not allocate at
// all.  For them this entry point takes only inputs and outputs and keeps
// its scratch -- the workspace status word and the per-CTA top-k candidate
// buffers -- in one fixed array compiled into the library.
//
// Limits and rules:
//   * The array is kNoAllocScratchBytes (32 MiB).  Every GPU that loads the
//     library holds it until the process exits.
//   * The fused kernel's grid is capped to the CTAs whose candidate
//     buffers fit in the array (63 CTAs at H_I = 32, top-2048), so large
//     problems run, more slowly than with a full workspace.  A problem whose
//     single CTA needs more than the array is rejected.
//   * All calls share the array and it keeps the last call's contents; each
//     call clears the status word it needs at zero.  Calls that overlap on
//     the GPU (different streams, or host threads on the same device) race
//     on it: serialise them.
//   * The first call on each device looks up the array's device address
//     with cudaGetSymbolAddress; make that first call before any stream
//     capture begins.
//   * Device-side status (timeouts) is written to the array's status word
//     and cleared by the next call; it is not reported by this entry point.
//   * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cstdio>
#include <mutex>
#include <string>

#include "dsa_common.cuh"

namespace dsa {
size_t indexer_workspace_bytes(int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int dtype,
                               int num_sms);
cudaError_t launch_indexer(const void* q, const float* q_scale, const void* k, const float* k_scale,
                           const float* w, int dtype, int B, int n_q, int q_pos0, int n_kv, int H, int d,
                           int topk, int* idx_out, float* scores_out, void* ws, size_t ws_bytes, int num_sms,
                           cudaStream_t stream);
int set_last_error(int code, const char* msg);  // message for dsa_last_error()
}  // namespace dsa

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

int set_err(int code, const std::string& msg) { return dsa::set_last_error(code, msg.c_str()); }

// Device address of the array on the current device (looked up once per device).
int scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_err(DSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return set_err(DSA_ERR_UNSUPPORTED, "device ordinal too large");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return set_err(DSA_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return DSA_OK;
}

}  // namespace

extern "C" DSA_API int idx_score_topk_noalloc(const void* q_I, const float* q_scale, const void* k_I,
                                              const float* k_scale, const float* w, int dtype, int B, int n_q,
                                              int q_pos0, int n_kv, int H_I, int d_I, int topk,
                                              int32_t* idx_out, void* stream) {
    // Shape validation is the same as idx_score_topk's (this query allocates nothing).
    size_t full = 0;
    int rc = idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, &full);
    if (rc) return rc;  // dsa_last_error() already holds the reason
    if (!q_I || !k_I || !w || !idx_out) return set_err(DSA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (dtype == DSA_E4M3 && (!q_scale || !k_scale))
        return set_err(DSA_ERR_INVALID_ARG, "e4m3 indexer needs q_scale and k_scale");
    if ((reinterpret_cast<uintptr_t>(q_I) | reinterpret_cast<uintptr_t>(k_I)) & 15u)
        return set_err(DSA_ERR_INVALID_ARG, "q_I and k_I must be 16-byte aligned");
    // Candidate bytes of one CTA; the grid is capped to what the array holds.
    const size_t per_cta = dsa::indexer_workspace_bytes(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, 1);
    const size_t room = kNoAllocScratchBytes - dsa::kWsHeaderBytes;
    if (per_cta > room) {
        char msg[160];
        snprintf(msg, sizeof(msg), "one CTA needs %zu scratch bytes; the no-alloc array holds %zu", per_cta, room);
        return set_err(DSA_ERR_UNSUPPORTED, msg);
    }
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return set_err(DSA_ERR_CUDA, std::string("device query: ") + cudaGetErrorString(e));
    const size_t fit = room / per_cta;
    int max_ctas = static_cast<int>(fit < static_cast<size_t>(sms) ? fit : static_cast<size_t>(sms));
    // The estimate above is exact for the prefill kernel, whose scratch grows with its grid.  The
    // one-query decode route sizes its selection scratch (slices per row) by the SM count it is
    // given, so check the bytes the launch will really use and shrink the grid until they fit.
    while (max_ctas > 1 &&
           dsa::indexer_workspace_bytes(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, max_ctas) > room)
        --max_ctas;
    if (dsa::indexer_workspace_bytes(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, max_ctas) > room) {
        char msg[160];
        snprintf(msg, sizeof(msg), "the problem needs more than the %zu scratch bytes of the no-alloc array", room);
        return set_err(DSA_ERR_UNSUPPORTED, msg);
    }
    void* scratch = nullptr;
    if ((rc = scratch_address(&scratch))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    e = cudaMemsetAsync(scratch, 0, dsa::kWsHeaderBytes, s);  // the status word must start at zero
    if (e != cudaSuccess) return set_err(DSA_ERR_CUDA, std::string("clear status: ") + cudaGetErrorString(e));
    e = dsa::launch_indexer(q_I, q_scale, k_I, k_scale, w, dtype, B, n_q, q_pos0, n_kv, H_I, d_I, topk, idx_out,
                            nullptr, scratch, kNoAllocScratchBytes, max_ctas, s);
    if (e != cudaSuccess) return set_err(DSA_ERR_CUDA, std::string("idx_score_topk_noalloc: ") + cudaGetErrorString(e));
    return DSA_OK;
}
