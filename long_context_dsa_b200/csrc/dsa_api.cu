// dsa_api.cu -- the C ABI of libdsa.so (declared in include/dsa.h).
//
// Host-side validation, workspace sizing, the index-cache descriptor and
// the layer-group loop.  Every compute step is a kernel launched from
// here; nothing is computed on the host.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "dsa_common.cuh"

namespace dsa {
// kernels (defined in the other translation units)
cudaError_t launch_topk_scores(const float* scores, int rows, int q_pos0, int n_kv, long long ld, int k, int* out,
                               WsHeader* hdr, int num_sms, cudaStream_t stream);
cudaError_t launch_sparse_attn(const void* Q, const void* K, const void* V, const int* idx, int B, int n_q,
                               int n_kv, int Hq, int Hkv, int d, int topk, float scale, void* O, bool out_bf16,
                               IdxShare share, KvPages pg, WsHeader* hdr, int num_sms, cudaStream_t stream);
cudaError_t launch_sparse_attn_fp8_paged(const void* Q, const void* K8, const float* k_scale, const void* V8,
                                         const float* v_scale, const int* idx, int B, int Hq, int Hkv, int d, int topk,
                                         float scale, void* O, bool out_bf16, KvPages pg, WsHeader* hdr, int num_sms,
                                         cudaStream_t stream);
cudaError_t launch_indexer_decode_paged(const void* q, const void* k_pages, const int* page_table, const int* seq_lens,
                                        const float* w, int B, int max_len, int page_size, int num_pages,
                                        int max_pages, int H, int topk, int* idx_out, void* ws, int num_sms,
                                        cudaStream_t stream);
size_t indexer_decode_workspace_bytes(int B, int q_pos0, int topk, int num_sms, bool varlen);
cudaError_t launch_sparse_attn_latent(const void* Q, const void* KV, const int* idx, int B, int n_q, int n_kv,
                                      int Hq, int topk, float scale, void* O, bool out_bf16, IdxShare share,
                                      WsHeader* hdr, int num_sms, cudaStream_t stream);
size_t indexer_workspace_bytes(int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int dtype,
                               int num_sms);
cudaError_t launch_overlap_count(const int* a, const int* b, long long rows, int k, int* out, int num_sms,
                                 cudaStream_t stream);
void greedy_pattern(const double* ov, int n, int n_f, char* out);
size_t sparse_attn_part_bytes(int B, int n_q, int Hq, int Hkv, int d, int topk, int num_sms);
size_t sparse_attn_latent_part_bytes(int B, int n_q, int Hq, int topk, int num_sms);
cudaError_t launch_indexer(const void* q, const float* q_scale, const void* k, const float* k_scale,
                           const float* w, int dtype, int B, int n_q, int q_pos0, int n_kv, int H, int d,
                           int topk, int* idx_out, float* scores_out, void* ws, size_t ws_bytes, int num_sms,
                           cudaStream_t stream);
}  // namespace dsa

using namespace dsa;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    if (e == cudaErrorNotSupported) return fail(DSA_ERR_UNSUPPORTED, "%s: no kernel for this shape", what);
    return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int sm_count(int* n) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t topk_scores_ws() { return kWsHeaderBytes; }

int check_ws(void* ws, size_t have, size_t need) {
    if (!ws) return fail(DSA_ERR_INVALID_ARG, "workspace is NULL");
    if (!aligned16(ws)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    if (have < need) return fail(DSA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", have, need);
    return DSA_OK;
}

int check_indexer_shape(int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int dtype) {
    if (B < 1 || n_q < 1 || q_pos0 < 0 || n_kv < 1)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes B=%d n_q=%d q_pos0=%d n_kv=%d", B, n_q, q_pos0, n_kv);
    if (static_cast<long long>(q_pos0) + n_q > n_kv)
        return fail(DSA_ERR_INVALID_ARG, "n_kv (%d) < q_pos0 + n_q (%d)", n_kv, q_pos0 + n_q);
    if (topk < 1) return fail(DSA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", topk);
    if (topk > DSA_TOPK_MAX) return fail(DSA_ERR_UNSUPPORTED, "topk %d > %d", topk, DSA_TOPK_MAX);
    if (dtype != DSA_BF16 && dtype != DSA_E4M3) return fail(DSA_ERR_INVALID_ARG, "indexer dtype must be BF16 or E4M3");
    if (!(H == 4 || H == 8 || H == 16 || H == 32 || H == 64))
        return fail(DSA_ERR_UNSUPPORTED, "H_I=%d not in {4,8,16,32,64}", H);
    if (!(d == 64 || d == 128)) return fail(DSA_ERR_UNSUPPORTED, "d_I=%d not in {64,128}", d);
    if (static_cast<long long>(B) * n_kv >= (1ll << 31) || static_cast<long long>(B) * n_q * H >= (1ll << 31))
        return fail(DSA_ERR_UNSUPPORTED, "problem too large for 32-bit row coordinates");
    return DSA_OK;
}

int check_attn_shape(const void* V, int B, int n_q, int n_kv, int Hq, int Hkv, int d_qk, int d_v, int topk) {
    if (B < 1 || n_q < 1 || n_kv < 1 || topk < 1 || Hq < 1 || Hkv < 1)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes B=%d n_q=%d n_kv=%d Hq=%d Hkv=%d topk=%d", B, n_q, n_kv, Hq, Hkv,
                    topk);
    if (Hq % Hkv != 0) return fail(DSA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (V == nullptr) {
        if (!(d_qk == 576 && d_v == 512 && Hkv == 1))
            return fail(DSA_ERR_UNSUPPORTED, "latent form needs d_qk=576, d_v=512, Hkv=1");
        if (Hq % 8 != 0) return fail(DSA_ERR_UNSUPPORTED, "latent form needs Hq a multiple of 8");
        return DSA_OK;
    }
    if (d_qk != d_v) return fail(DSA_ERR_UNSUPPORTED, "d_qk != d_v needs the latent form");
    if (!(d_qk == 64 || d_qk == 128)) return fail(DSA_ERR_UNSUPPORTED, "head dim %d not in {64,128}", d_qk);
    if (Hq / Hkv > 8) return fail(DSA_ERR_UNSUPPORTED, "GQA group %d > 8", Hq / Hkv);
    return DSA_OK;
}

}  // namespace

namespace dsa {
// Lets other translation units of the library report through dsa_last_error().
int set_last_error(int code, const char* msg) {
    g_last_error = msg ? msg : "";
    return code;
}
}  // namespace dsa

extern "C" {

const char* dsa_last_error(void) { return g_last_error.c_str(); }

int dsa_version(void) { return 100; }

int dsa_check_status(void* workspace, void* stream, int* bits) {
    if (!workspace) return fail(DSA_ERR_INVALID_ARG, "workspace is NULL");
    WsHeader h;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(int) * 2, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(int) * 2, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "dsa_check_status");
    if (bits) *bits = h.status;
    if (h.status & DSA_STATUS_TIMEOUT)
        return fail(DSA_ERR_TIMEOUT, "a device wait timed out (site 0x%x)", h.detail);
    if (h.status) return fail(DSA_ERR_DEVICE, "device status 0x%x (detail %d)", h.status, h.detail);
    return DSA_OK;
}

int dsa_reset_status(void* workspace, void* stream) {
    if (!workspace) return fail(DSA_ERR_INVALID_ARG, "workspace is NULL");
    cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeaderBytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dsa_reset_status");
    return DSA_OK;
}

// --------------------------------------------------------------- top-k alone
int idx_topk_scores_workspace_size(int rows, int q_pos0, int n_kv, int topk, size_t* bytes) {
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    if (rows < 1 || q_pos0 < 0 || n_kv < 1 || static_cast<long long>(q_pos0) + rows > n_kv)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes rows=%d q_pos0=%d n_kv=%d", rows, q_pos0, n_kv);
    if (topk < 1) return fail(DSA_ERR_INVALID_ARG, "topk must be >= 1");
    if (topk > DSA_TOPK_MAX) return fail(DSA_ERR_UNSUPPORTED, "topk %d > %d", topk, DSA_TOPK_MAX);
    *bytes = topk_scores_ws();
    return DSA_OK;
}

int idx_topk_scores(const float* scores, int rows, int q_pos0, int n_kv, int64_t ld, int topk, int32_t* idx_out,
                    void* workspace, size_t workspace_bytes, void* stream) {
    size_t need;
    int rc = idx_topk_scores_workspace_size(rows, q_pos0, n_kv, topk, &need);
    if (rc) return rc;
    if (!scores || !idx_out) return fail(DSA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (ld < n_kv) return fail(DSA_ERR_INVALID_ARG, "ld (%lld) < n_kv (%d)", static_cast<long long>(ld), n_kv);
    if ((rc = check_ws(workspace, workspace_bytes, need))) return rc;
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    cudaError_t e = launch_topk_scores(scores, rows, q_pos0, n_kv, ld, topk, idx_out,
                                       static_cast<WsHeader*>(workspace), sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "idx_topk_scores");
    return DSA_OK;
}

// ------------------------------------------------------- fused indexer top-k
int idx_score_topk_workspace_size(int B, int n_q, int q_pos0, int n_kv, int H_I, int d_I, int topk, int dtype,
                                  size_t* bytes) {
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    int rc = check_indexer_shape(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype);
    if (rc) return rc;
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    *bytes = kWsHeaderBytes + indexer_workspace_bytes(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, sms);
    return DSA_OK;
}

int idx_score_topk(const void* q_I, const float* q_scale, const void* k_I, const float* k_scale, const float* w,
                   int dtype, int B, int n_q, int q_pos0, int n_kv, int H_I, int d_I, int topk, int32_t* idx_out,
                   void* workspace, size_t workspace_bytes, void* stream) {
    size_t need;
    int rc = idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, &need);
    if (rc) return rc;
    if (!q_I || !k_I || !w || !idx_out) return fail(DSA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (dtype == DSA_E4M3 && (!q_scale || !k_scale))
        return fail(DSA_ERR_INVALID_ARG, "e4m3 indexer needs q_scale and k_scale");
    if (!aligned16(q_I) || !aligned16(k_I)) return fail(DSA_ERR_INVALID_ARG, "q_I and k_I must be 16-byte aligned");
    if ((rc = check_ws(workspace, workspace_bytes, need))) return rc;
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    cudaError_t e = launch_indexer(q_I, q_scale, k_I, k_scale, w, dtype, B, n_q, q_pos0, n_kv, H_I, d_I, topk,
                                   idx_out, nullptr, workspace, workspace_bytes, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "idx_score_topk");
    return DSA_OK;
}

int idx_scores(const void* q_I, const float* q_scale, const void* k_I, const float* k_scale, const float* w,
               int dtype, int B, int n_q, int q_pos0, int n_kv, int H_I, int d_I, float* scores, void* workspace,
               size_t workspace_bytes, void* stream) {
    int rc = check_indexer_shape(B, n_q, q_pos0, n_kv, H_I, d_I, 1, dtype);
    if (rc) return rc;
    if (!q_I || !k_I || !w || !scores) return fail(DSA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (dtype == DSA_E4M3 && (!q_scale || !k_scale))
        return fail(DSA_ERR_INVALID_ARG, "e4m3 indexer needs q_scale and k_scale");
    if (!aligned16(q_I) || !aligned16(k_I)) return fail(DSA_ERR_INVALID_ARG, "q_I and k_I must be 16-byte aligned");
    if ((rc = check_ws(workspace, workspace_bytes, kWsHeaderBytes))) return rc;
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    cudaError_t e = launch_indexer(q_I, q_scale, k_I, k_scale, w, dtype, B, n_q, q_pos0, n_kv, H_I, d_I, 1, nullptr,
                                   scores, workspace, workspace_bytes, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "idx_scores");
    return DSA_OK;
}

// ------------------------------------------------------------- index cache
int idx_cache_init(dsa_index_cache* cache, int32_t* buf, int64_t rows, int topk) {
    if (!cache || !buf) return fail(DSA_ERR_INVALID_ARG, "NULL cache or buffer");
    if (rows < 1 || topk < 1) return fail(DSA_ERR_INVALID_ARG, "bad cache shape");
    cache->buf = buf;
    cache->rows = rows;
    cache->topk = topk;
    cache->writer = -1;
    cache->valid = 0;
    return DSA_OK;
}

static int pattern_check(const char* pattern, int n_layers) {
    if (!pattern) return fail(DSA_ERR_INVALID_ARG, "pattern is NULL");
    const int n = static_cast<int>(strnlen(pattern, 4096));
    if (n == 0 || pattern[0] != 'F') return fail(DSA_ERR_INVALID_ARG, "pattern must start with F");
    for (int i = 0; i < n; ++i)
        if (pattern[i] != 'F' && pattern[i] != 'S')
            return fail(DSA_ERR_INVALID_ARG, "pattern may only hold F and S (got '%c' at %d)", pattern[i], i);
    if (n_layers >= 0 && n != n_layers)
        return fail(DSA_ERR_INVALID_ARG, "pattern length %d != n_layers %d", n, n_layers);
    return DSA_OK;
}

int idx_cache_put(dsa_index_cache* cache, int layer, const char* pattern) {
    if (!cache) return fail(DSA_ERR_INVALID_ARG, "cache is NULL");
    int rc = pattern_check(pattern, -1);
    if (rc) return rc;
    if (layer < 0 || layer >= static_cast<int>(strlen(pattern)) || pattern[layer] != 'F')
        return fail(DSA_ERR_INVALID_ARG, "layer %d is not an F layer", layer);
    cache->writer = layer;
    cache->valid = 1;
    return DSA_OK;
}

int idx_cache_get(const dsa_index_cache* cache, int layer, const char* pattern, const int32_t** idx) {
    if (!cache || !idx) return fail(DSA_ERR_INVALID_ARG, "NULL argument");
    int rc = pattern_check(pattern, -1);
    if (rc) return rc;
    if (layer < 0 || layer >= static_cast<int>(strlen(pattern))) return fail(DSA_ERR_INVALID_ARG, "layer out of range");
    int last_f = -1;
    for (int i = 0; i <= layer; ++i)
        if (pattern[i] == 'F') last_f = i;
    if (!cache->valid || cache->writer != last_f)
        return fail(DSA_ERR_INVALID_ARG, "layer %d needs indices from F layer %d, which has not written the cache",
                    layer, last_f);
    *idx = cache->buf;
    return DSA_OK;
}

// ------------------------------------------------------------ F/S pattern search
int idx_overlap(const int32_t* idx_a, const int32_t* idx_b, int64_t rows, int topk, int32_t* counts,
                void* stream) {
    if (!idx_a || !idx_b || !counts) return fail(DSA_ERR_INVALID_ARG, "NULL pointer");
    if (rows < 1 || topk < 1) return fail(DSA_ERR_INVALID_ARG, "bad sizes rows=%lld topk=%d",
                                          static_cast<long long>(rows), topk);
    int sms;
    int rc = sm_count(&sms);
    if (rc) return rc;
    cudaError_t e = launch_overlap_count(idx_a, idx_b, rows, topk, counts, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "idx_overlap");
    return DSA_OK;
}

int layer_pattern_search(const double* overlap, int n_layers, int n_f, char* pattern_out) {
    if (!overlap || !pattern_out) return fail(DSA_ERR_INVALID_ARG, "NULL pointer");
    if (n_layers < 1 || n_layers > 4096) return fail(DSA_ERR_INVALID_ARG, "n_layers %d out of range", n_layers);
    if (n_f < 1 || n_f > n_layers) return fail(DSA_ERR_INVALID_ARG, "n_f %d not in [1, %d]", n_f, n_layers);
    for (int f = 0; f < n_layers; ++f)
        for (int j = f + 1; j < n_layers; ++j) {
            const double v = overlap[static_cast<size_t>(f) * n_layers + j];
            if (!(v >= 0.0 && v <= 1.0)) return fail(DSA_ERR_INVALID_ARG, "overlap[%d][%d] not in [0, 1]", f, j);
        }
    greedy_pattern(overlap, n_layers, n_f, pattern_out);
    return DSA_OK;
}

// ------------------------------------------------------------ sparse attention
int sparse_attn_topk_workspace_size(int B, int n_q, int n_kv, int Hq, int Hkv, int d_qk, int d_v, int topk,
                                    size_t* bytes) {
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    if (B < 1 || n_q < 1 || n_kv < 1 || Hq < 1 || Hkv < 1 || d_qk < 1 || d_v < 1 || topk < 1)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes");
    size_t part = 0;
    if (d_qk == d_v && Hkv > 0 && Hq % Hkv == 0) {
        int sms;
        int rc = sm_count(&sms);
        if (rc) return rc;
        part = sparse_attn_part_bytes(B, n_q, Hq, Hkv, d_qk, topk, sms);
    } else if (d_qk == 576 && d_v == 512 && Hkv == 1) {  // the latent form
        int sms;
        int rc = sm_count(&sms);
        if (rc) return rc;
        part = sparse_attn_latent_part_bytes(B, n_q, Hq, topk, sms);
    }
    *bytes = kWsHeaderBytes + part;
    return DSA_OK;
}

namespace {
int attn_common(const void* Q, const void* K, const void* V, const int32_t* idx, int B, int n_q, int n_kv, int Hq,
                int Hkv, int d_qk, int d_v, int topk, float scale, void* O, int o_dtype, dsa::IdxShare share,
                void* workspace, size_t workspace_bytes, void* stream, dsa::KvPages pages = dsa::kContiguous) {
    int rc = check_attn_shape(V, B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk);
    if (rc) return rc;
    if (!Q || !K || !idx || !O) return fail(DSA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (o_dtype != DSA_F32 && o_dtype != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "o_dtype must be F32 or BF16");
    if (!aligned16(Q) || !aligned16(K) || (V && !aligned16(V)))
        return fail(DSA_ERR_INVALID_ARG, "Q, K, V must be 16-byte aligned");
    size_t need;
    if ((rc = sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk, &need))) return rc;
    if ((rc = check_ws(workspace, workspace_bytes, need))) return rc;
    if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(d_qk));
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    cudaError_t e;
    if (V == nullptr && pages.table) return fail(DSA_ERR_UNSUPPORTED, "paged caches need the separate K/V form");
    if (V == nullptr)
        e = launch_sparse_attn_latent(Q, K, idx, B, n_q, n_kv, Hq, topk, scale, O, o_dtype == DSA_BF16, share,
                                      static_cast<WsHeader*>(workspace), sms, static_cast<cudaStream_t>(stream));
    else
        e = launch_sparse_attn(Q, K, V, idx, B, n_q, n_kv, Hq, Hkv, d_qk, topk, scale, O, o_dtype == DSA_BF16,
                               share, pages, static_cast<WsHeader*>(workspace), sms,
                               static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "sparse_attn_topk");
    return DSA_OK;
}
}  // namespace

int sparse_attn_topk(const void* Q, const void* K, const void* V, const int32_t* idx, int B, int n_q, int n_kv,
                     int Hq, int Hkv, int d_qk, int d_v, int topk, float scale, void* O, int o_dtype,
                     void* workspace, size_t workspace_bytes, void* stream) {
    return attn_common(Q, K, V, idx, B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk, scale, O, o_dtype, dsa::kNoShare,
                       workspace, workspace_bytes, stream);
}

int sparse_attn_topk_paged(const void* Q, const void* K_pages, const void* V_pages, const int32_t* page_table,
                           const int32_t* seq_lens, const int32_t* idx, int B, int page_size, int num_pages,
                           int max_pages, int Hq, int Hkv, int d, int topk, float scale, void* O, int o_dtype,
                           void* workspace, size_t workspace_bytes, void* stream) {
    if (!page_table || !seq_lens || !V_pages) return fail(DSA_ERR_INVALID_ARG, "NULL page table, lengths or V");
    if (page_size < 1 || num_pages < 1 || max_pages < 1)
        return fail(DSA_ERR_INVALID_ARG, "bad page geometry page_size=%d num_pages=%d max_pages=%d", page_size,
                    num_pages, max_pages);
    const long long pool = static_cast<long long>(num_pages) * page_size;
    if (pool > 0x7fffffffll) return fail(DSA_ERR_INVALID_ARG, "page pool too large");
    const dsa::KvPages pages = {page_table, seq_lens, page_size, max_pages, num_pages, dsa::page_shift_of(page_size)};
    return attn_common(Q, K_pages, V_pages, idx, B, 1, static_cast<int>(pool), Hq, Hkv, d, d, topk, scale, O,
                       o_dtype, dsa::kNoShare, workspace, workspace_bytes, stream, pages);
}

int sparse_attn_topk_paged_e4m3(const void* Q, const void* K8_pages, const float* k_scale, const void* V8_pages,
                                const float* v_scale, const int32_t* page_table, const int32_t* seq_lens,
                                const int32_t* idx, int B, int page_size, int num_pages, int max_pages, int Hq, int Hkv,
                                int d, int topk, float scale, void* O, int o_dtype, void* workspace,
                                size_t workspace_bytes, void* stream) {
    if (!Q || !K8_pages || !k_scale || !V8_pages || !v_scale || !page_table || !seq_lens || !idx || !O)
        return fail(DSA_ERR_INVALID_ARG, "NULL pointer");
    if (page_size < 1 || num_pages < 1 || max_pages < 1)
        return fail(DSA_ERR_INVALID_ARG, "bad page geometry page_size=%d num_pages=%d max_pages=%d", page_size,
                    num_pages, max_pages);
    const long long pool = static_cast<long long>(num_pages) * page_size;
    if (pool > 0x7fffffffll) return fail(DSA_ERR_INVALID_ARG, "page pool too large");
    int rc = check_attn_shape(V8_pages, B, 1, static_cast<int>(pool), Hq, Hkv, d, d, topk);
    if (rc) return rc;
    if (o_dtype != DSA_F32 && o_dtype != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "o_dtype must be F32 or BF16");
    if (!aligned16(Q) || !aligned16(K8_pages) || !aligned16(V8_pages))
        return fail(DSA_ERR_INVALID_ARG, "Q, K8_pages, V8_pages must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(k_scale) | reinterpret_cast<uintptr_t>(v_scale)) & 3u)
        return fail(DSA_ERR_INVALID_ARG, "scales must be 4-byte aligned");
    size_t need;
    if ((rc = sparse_attn_topk_workspace_size(B, 1, static_cast<int>(pool), Hq, Hkv, d, d, topk, &need))) return rc;
    if ((rc = check_ws(workspace, workspace_bytes, need))) return rc;
    if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(d));
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    const dsa::KvPages pages = {page_table, seq_lens, page_size, max_pages, num_pages, dsa::page_shift_of(page_size)};
    cudaError_t e = launch_sparse_attn_fp8_paged(Q, K8_pages, k_scale, V8_pages, v_scale, idx, B, Hq, Hkv, d, topk,
                                                 scale, O, o_dtype == DSA_BF16, pages,
                                                 static_cast<WsHeader*>(workspace), sms,
                                                 static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "sparse_attn_topk_paged_e4m3");
    return DSA_OK;
}

int idx_score_topk_paged_workspace_size(int B, int max_seq_len, int H_I, int d_I, int topk, size_t* bytes) {
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    if (B < 1 || max_seq_len < 1 || topk < 1 || topk > DSA_TOPK_MAX)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes");
    if (!((H_I == 32 || H_I == 64) && d_I == 128))
        return fail(DSA_ERR_UNSUPPORTED, "paged decode indexer supports H_I in {32, 64}, d_I = 128");
    int sms;
    int rc = sm_count(&sms);
    if (rc) return rc;
    *bytes = kWsHeaderBytes + indexer_decode_workspace_bytes(B, max_seq_len - 1, topk, sms, true);
    return DSA_OK;
}

int idx_score_topk_paged(const void* q_I, const void* k_pages, const int32_t* page_table, const int32_t* seq_lens,
                         const float* w, int B, int max_seq_len, int page_size, int num_pages, int max_pages,
                         int H_I, int d_I, int topk, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                         void* stream) {
    if (!q_I || !k_pages || !page_table || !seq_lens || !w || !idx_out) return fail(DSA_ERR_INVALID_ARG, "NULL pointer");
    if (page_size < 16 || (page_size & (page_size - 1)) != 0)
        return fail(DSA_ERR_INVALID_ARG, "page_size %d must be a power of two >= 16", page_size);
    if (num_pages < 1 || max_pages < 1 || static_cast<long long>(max_pages) * page_size < max_seq_len)
        return fail(DSA_ERR_INVALID_ARG, "page table cannot hold max_seq_len tokens");
    if (static_cast<long long>(num_pages) * page_size > 0x7fffffffll) return fail(DSA_ERR_INVALID_ARG, "page pool too large");
    if (!aligned16(q_I) || !aligned16(k_pages)) return fail(DSA_ERR_INVALID_ARG, "q_I and k_pages must be 16-byte aligned");
    size_t need;
    int rc = idx_score_topk_paged_workspace_size(B, max_seq_len, H_I, d_I, topk, &need);
    if (rc) return rc;
    if ((rc = check_ws(workspace, workspace_bytes, need))) return rc;
    int sms;
    if ((rc = sm_count(&sms))) return rc;
    cudaError_t e = launch_indexer_decode_paged(q_I, k_pages, page_table, seq_lens, w, B, max_seq_len, page_size,
                                                num_pages, max_pages, H_I, topk, idx_out, workspace, sms,
                                                static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "idx_score_topk_paged");
    return DSA_OK;
}

int sparse_attn_topk_shared(const void* Q, const void* K, const void* V, const int32_t* idx, int B, int n_q,
                            int q_pos0, int n_kv, int Hq, int Hkv, int d_qk, int d_v, int topk, int q_per_idx,
                            float scale, void* O, int o_dtype, void* workspace, size_t workspace_bytes,
                            void* stream) {
    if (q_per_idx < 1) return fail(DSA_ERR_INVALID_ARG, "q_per_idx must be >= 1");
    if (q_pos0 < 0 || static_cast<long long>(q_pos0) + n_q > n_kv)
        return fail(DSA_ERR_INVALID_ARG, "query positions q_pos0..q_pos0+n_q-1 must lie inside the cache");
    const dsa::IdxShare share = {q_per_idx, q_pos0, 1};
    return attn_common(Q, K, V, idx, B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk, scale, O, o_dtype, share, workspace,
                       workspace_bytes, stream);
}

// ------------------------------------------------------------- layer group
int layer_group_forward_workspace_size(const dsa_group_shape* sh, size_t* bytes) {
    if (!sh || !bytes) return fail(DSA_ERR_INVALID_ARG, "NULL argument");
    size_t a = 0, b = 0;
    int rc = idx_score_topk_workspace_size(sh->B, sh->n_q, sh->q_pos0, sh->n_kv, sh->H_I, sh->d_I, sh->topk,
                                           sh->idx_dtype, &a);
    if (rc) return rc;
    if ((rc = sparse_attn_topk_workspace_size(sh->B, sh->n_q, sh->n_kv, sh->Hq, sh->Hkv, sh->d_qk, sh->d_v,
                                              sh->topk, &b)))
        return rc;
    *bytes = a > b ? a : b;
    return DSA_OK;
}

int layer_group_forward(const dsa_group_shape* sh, const dsa_layer_args* layers, int n_layers, const char* pattern,
                        dsa_index_cache* cache, dsa_group_stats* stats, void* workspace, size_t workspace_bytes,
                        void* stream) {
    if (!sh || !layers || !cache) return fail(DSA_ERR_INVALID_ARG, "NULL argument");
    if (n_layers < 1) return fail(DSA_ERR_INVALID_ARG, "n_layers must be >= 1");
    int rc = pattern_check(pattern, n_layers);
    if (rc) return rc;
    if (!cache->buf || cache->rows != static_cast<int64_t>(sh->B) * sh->n_q || cache->topk != sh->topk)
        return fail(DSA_ERR_INVALID_ARG, "cache buffer does not match B*n_q x topk");
    size_t need;
    if ((rc = layer_group_forward_workspace_size(sh, &need))) return rc;
    if ((rc = check_ws(workspace, workspace_bytes, need))) return rc;
    // validate every layer before launching anything
    for (int l = 0; l < n_layers; ++l) {
        const dsa_layer_args& L = layers[l];
        if (!L.Q || !L.K || !L.O) return fail(DSA_ERR_INVALID_ARG, "layer %d: NULL attention tensor", l);
        if (pattern[l] == 'F' && (!L.q_I || !L.k_I || !L.w))
            return fail(DSA_ERR_INVALID_ARG, "layer %d (F): NULL indexer tensor", l);
        if ((rc = check_attn_shape(L.V, sh->B, sh->n_q, sh->n_kv, sh->Hq, sh->Hkv, sh->d_qk, sh->d_v, sh->topk)))
            return rc;
    }
    if (stats) stats->indexer_launches = stats->attention_launches = 0;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    auto mark = [&](int i) -> int {
        if (!stats || !stats->events) return DSA_OK;
        cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(stats->events[i]), cs);
        return e == cudaSuccess ? DSA_OK : cuda_fail(e, "layer_group_forward event");
    };
    cache->valid = 0;
    cache->writer = -1;
    for (int l = 0; l < n_layers; ++l) {
        const dsa_layer_args& L = layers[l];
        if ((rc = mark(3 * l))) return rc;
        if (pattern[l] == 'F') {  // the one extra branch: only F layers run the indexer
            rc = idx_score_topk(L.q_I, L.q_scale, L.k_I, L.k_scale, L.w, sh->idx_dtype, sh->B, sh->n_q, sh->q_pos0,
                                sh->n_kv, sh->H_I, sh->d_I, sh->topk, cache->buf, workspace, workspace_bytes, stream);
            if (rc) return rc;
            if ((rc = idx_cache_put(cache, l, pattern))) return rc;
            if (stats) stats->indexer_launches++;
        }
        if ((rc = mark(3 * l + 1))) return rc;
        const int32_t* idx = nullptr;
        if ((rc = idx_cache_get(cache, l, pattern, &idx))) return rc;
        rc = sparse_attn_topk(L.Q, L.K, L.V, idx, sh->B, sh->n_q, sh->n_kv, sh->Hq, sh->Hkv, sh->d_qk, sh->d_v,
                              sh->topk, sh->scale, L.O, sh->o_dtype, workspace, workspace_bytes, stream);
        if (rc) return rc;
        if (stats) stats->attention_launches++;
        if ((rc = mark(3 * l + 2))) return rc;
    }
    return DSA_OK;
}

}  // extern "C"
