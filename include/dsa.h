/*
 * dsa.h -- C ABI of libdsa.so: the DeepSeek-Sparse-Attention-style token
 * indexer with cross-layer index reuse (IndexCache F/S layers; IndexShare,
 * one indexer per four layers), for NVIDIA B200 (sm_100a).
 *
 * Sources the operations follow (Chinese web pages, cited by title and
 * section):
 *   [QbitAI]    QbitAI article on IndexCache (app.myzaker.com), sections
 *               "IndexCache" and "GLM-5.2 已经用过了".
 *   [Term]      earlyterms.com term page "IndexShare", definition.
 *   [Explainer] "IndexShare 技术解读：4 层共享 indexer 如何把计算成本砍到三分之一"
 *               (yun88.com), sections "稀疏注意力的隐性开销：indexer" and
 *               "IndexShare 的共享机制：每 4 层一个 indexer".
 *   [Linkstar]  "20万token压进10秒，清华这波操作让AI算力成本直接砍半"
 *               (linkstar.cloud), sections on DSA's cost and on F/S layers
 *               ("'偷懒'的艺术：相邻层其实在重复劳动").
 *
 * Conventions for every entry point:
 *   - Return value is a status code (DSA_OK == 0).  No C++ exception
 *     crosses the ABI and no kernel traps; device-detected errors are
 *     recorded in the workspace status word and returned by
 *     dsa_check_status().
 *   - Tensor arguments are DEVICE pointers owned by the caller, row-major
 *     and contiguous in the stated layout.  The library never allocates
 *     or frees device memory and keeps no pointer after a call returns.
 *   - Scratch memory is a caller-owned device `workspace` of at least the
 *     size the matching *_workspace_size() query reports.  Its first 256
 *     bytes are the status word; calls that share a workspace must not
 *     overlap on the GPU.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream.
 *   - Shapes are validated on the host before any launch; a rejected call
 *     launches nothing and returns DSA_ERR_INVALID_ARG or
 *     DSA_ERR_UNSUPPORTED with a message in dsa_last_error().
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define DSA_OK               0
#define DSA_ERR_INVALID_ARG  1  /* bad shape, null pointer, bad pattern, small workspace */
#define DSA_ERR_UNSUPPORTED  2  /* valid request the library has no kernel for           */
#define DSA_ERR_CUDA         3  /* a CUDA runtime call or launch failed                  */
#define DSA_ERR_TIMEOUT      4  /* a bounded device-side wait gave up (status word)      */
#define DSA_ERR_DEVICE       5  /* a kernel rejected its data (status word), e.g. an
                                   index outside [-1, n_kv) or a NaN score               */

/* ---- element types --------------------------------------------------- */
#define DSA_BF16  0
#define DSA_E4M3  1   /* OCP fp8 E4M3 (bias 7, max 448, no infinities) */
#define DSA_F32   2

/* ---- device status word bits (dsa_check_status detail) ---------------- */
#define DSA_STATUS_TIMEOUT    0x1   /* a bounded wait expired                  */
#define DSA_STATUS_BAD_INDEX  0x2   /* sparse attention met an out-of-range idx */
#define DSA_STATUS_NAN_SCORE  0x4   /* top-k met a NaN score                    */
#define DSA_STATUS_OVERFLOW   0x8   /* a candidate buffer would have overflowed */

/* Test hook of the timeout path.  The 32-bit word at byte offset 8 of a
 * workspace (inside its status word) must be zero in normal use (a zeroed
 * workspace and dsa_reset_status() leave it so).  If it holds this value,
 * the TMA producers of idx_score_topk's kernels withhold the first key tile
 * of each CTA: every bounded wait on that tile runs out (about 2 s), the
 * kernel winds down without faulting and dsa_check_status() returns
 * DSA_ERR_TIMEOUT.  The indices written by such a call are meaningless. */
#define DSA_TEST_WITHHOLD_TILE 0x5D5A7E57

/* Largest top-k the library selects. */
#define DSA_TOPK_MAX 2048

/* Thread-local text of the last error raised on this host thread. */
DSA_API const char* dsa_last_error(void);

/* Library ABI version (major*100 + minor). */
DSA_API int dsa_version(void);

/* Read the workspace status word (synchronises `stream`), clear it, and map
 * it to a status code: DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE.  If
 * `bits` is non-NULL it receives the raw DSA_STATUS_* bits. */
DSA_API int dsa_check_status(void* workspace, void* stream, int* bits);

/* Zero the status word (asynchronous on `stream`). */
DSA_API int dsa_reset_status(void* workspace, void* stream);

/* ======================================================================
 * idx_score_topk -- indexer scores + per-row top-k, fused (F layers).
 *
 * Operation ([QbitAI] §IndexCache: a light indexer before each attention
 * layer picks the important tokens; [Term]: its work is "dot product +
 * top-k"; the form below is the DeepSeek-Sparse-Attention lightning
 * indexer):
 *     score[b,i,s] = sum_h w[b,i,h] * ReLU(q_I[b,i,h,:] . k_I[b,s,:])
 * for s = 0 .. q_pos0+i (query row i sits at absolute position q_pos0+i
 * and sees itself).  fp8: q_I and k_I are E4M3 codes whose real values
 * are code * q_scale[b,i,h] and code * k_scale[b,s].
 * Selection: the `topk` largest scores per row, ties to the lower token
 * index; a row with no more than `topk` candidates selects them all.
 * The L x L score matrix is never written to memory.
 *
 * Layouts:
 *   q_I     [B, n_q, H_I, d_I]  bf16 or e4m3 (dtype)
 *   q_scale [B, n_q, H_I]       fp32, e4m3 only (else NULL)
 *   k_I     [B, n_kv, d_I]      bf16 or e4m3
 *   k_scale [B, n_kv]           fp32, e4m3 only (else NULL)
 *   w       [B, n_q, H_I]       fp32
 *   idx_out [B, n_q, topk]      int32: selected token indices of each row
 *                               in ascending order, then -1 padding.
 * Requires n_kv >= q_pos0 + n_q, 1 <= topk <= DSA_TOPK_MAX,
 * H_I in {4, 8, 16, 32, 64}, d_I in {64, 128}.
 * ====================================================================== */
DSA_API int idx_score_topk_workspace_size(int B, int n_q, int q_pos0, int n_kv, int H_I, int d_I,
                                  int topk, int dtype, size_t* bytes);
DSA_API int idx_score_topk(const void* q_I, const float* q_scale, const void* k_I, const float* k_scale,
                   const float* w, int dtype, int B, int n_q, int q_pos0, int n_kv,
                   int H_I, int d_I, int topk, int32_t* idx_out,
                   void* workspace, size_t workspace_bytes, void* stream);

/* idx_scores -- the same indexer arithmetic without the selection: writes
 * scores [B, n_q, n_kv] fp32 for the key tiles the fused kernel visits
 * (s <= q_pos0+i exact, s > q_pos0+i within a visited tile -inf, other
 * entries untouched).  For checking the scores themselves; it writes the
 * full score matrix, so it is a test/debug path, not the product path.
 * Workspace: 256 bytes (status word). */
DSA_API int idx_scores(const void* q_I, const float* q_scale, const void* k_I, const float* k_scale,
                       const float* w, int dtype, int B, int n_q, int q_pos0, int n_kv,
                       int H_I, int d_I, float* scores, void* workspace, size_t workspace_bytes,
                       void* stream);

/* ======================================================================
 * idx_topk_scores -- the top-k selection alone, on a given score array.
 *
 * The same selection rule as idx_score_topk, from the same building blocks
 * (per-warp candidate buffers, radix select, merge of sorted sub-buffers);
 * it prunes with the exact radix select only, while the fused kernel first
 * prunes to a superset by a score histogram.  Given identical scores both
 * give identical indices; used to check a selection bit-exactly against a
 * reference on a score array.
 *   scores  [rows, ld] fp32 (row i uses columns 0 .. q_pos0+i; ld >= n_kv)
 *   idx_out [rows, topk] int32, layout as above.
 * Scores in the causal range must not be NaN (DSA_STATUS_NAN_SCORE).
 * ====================================================================== */
DSA_API int idx_topk_scores_workspace_size(int rows, int q_pos0, int n_kv, int topk, size_t* bytes);
DSA_API int idx_topk_scores(const float* scores, int rows, int q_pos0, int n_kv, int64_t ld, int topk,
                    int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream);

/* ======================================================================
 * Index cache -- one int32 [rows, topk] buffer per layer group.
 *
 * [Linkstar] F/S layers: F layers keep the indexer and store the selected
 * indices; S layers copy the most recent F layer's result and skip the
 * indexer.  [QbitAI] §IndexCache: no extra GPU memory.  The cache is a
 * host descriptor around ONE caller-owned device buffer; reading it
 * launches nothing and copies nothing.
 * ====================================================================== */
typedef struct dsa_index_cache {
    int32_t* buf;     /* caller-owned device buffer [rows, topk] */
    int64_t rows;     /* B * n_q                                 */
    int topk;
    int writer;       /* layer that last wrote buf, -1 if none   */
    int valid;        /* 1 once an F layer has written           */
} dsa_index_cache;

/* Bind `buf` to an empty cache. */
DSA_API int idx_cache_init(dsa_index_cache* cache, int32_t* buf, int64_t rows, int topk);
/* Record that F layer `layer` has (been enqueued to) write(n) the buffer. */
DSA_API int idx_cache_put(dsa_index_cache* cache, int layer, const char* pattern);
/* Device pointer of the indices layer `layer` must use: the buffer written
 * by the most recent F layer at or before `layer` in `pattern`.
 * DSA_ERR_INVALID_ARG if that F layer has not written it. */
DSA_API int idx_cache_get(const dsa_index_cache* cache, int layer, const char* pattern,
                  const int32_t** idx);

/* ======================================================================
 * sparse_attn_topk -- attention over each query's selected tokens.
 *
 * [Explainer] §稀疏注意力: each token attends only to its top-k history
 * tokens; §IndexShare 的共享机制: S layers reuse the indices with their own
 * attention weights, so every layer calls this with its own Q/K/V.
 *     O[b,i,h] = sum_{j in I[b,i]} softmax_j(scale * Q[b,i,h].K[b,j,g(h)]) V[b,j,g(h)]
 * g(h) = h / (Hq/Hkv).  Entries of idx equal to -1 are skipped; any other
 * value outside [0, n_kv) is skipped and flagged (DSA_STATUS_BAD_INDEX).
 *   Q   [B, n_q, Hq, d_qk]  bf16
 *   K   [B, n_kv, Hkv, d_qk] bf16
 *   V   [B, n_kv, Hkv, d_v]  bf16, or NULL for the latent form: one row per
 *       token (Hkv == 1) is the key (all d_qk dims) and the value (its
 *       first d_v dims).
 *   idx [B, n_q, topk] int32
 *   O   [B, n_q, Hq, d_v]   fp32 (o_dtype DSA_F32) or bf16 (DSA_BF16)
 * Supported: d_qk == d_v in {64, 128} with Hq/Hkv in {1,2,4,8};
 * latent d_qk = 576, d_v = 512, Hkv = 1, Hq a multiple of 8.
 * Workspace: the status word, plus (when B*n_q*Hkv is too small to occupy
 * every warp of the GPU, e.g. decode) fp32 partial softmax state for each
 * query head and range of the index list, merged by a second kernel.  The
 * size depends on the shape and the device's SM count only.
 * ====================================================================== */
DSA_API int sparse_attn_topk_workspace_size(int B, int n_q, int n_kv, int Hq, int Hkv, int d_qk, int d_v,
                                    int topk, size_t* bytes);
DSA_API int sparse_attn_topk(const void* Q, const void* K, const void* V, const int32_t* idx,
                     int B, int n_q, int n_kv, int Hq, int Hkv, int d_qk, int d_v, int topk,
                     float scale, void* O, int o_dtype,
                     void* workspace, size_t workspace_bytes, void* stream);

/* sparse_attn_topk_shared -- the same attention where consecutive query rows
 * share one index row (multi-token / speculative decode).
 *
 * [Term] §IndexShare: the sharing that lets layers reuse one indexer also
 * raised MTP speculative-decoding acceptance; this entry point lets several
 * query tokens of a sequence (a verified draft) reuse one F-layer selection.
 * Query row i of sequence b (absolute position q_pos0 + i) uses index row
 * idx[b, i / q_per_idx] and skips the entries of that row beyond its own
 * position, so a selection made for the group's last token serves every
 * token of the group causally.
 *   idx [B, ceil(n_q / q_per_idx), topk] int32; everything else as in
 *   sparse_attn_topk (workspace size from sparse_attn_topk_workspace_size
 *   with the same B, n_q).  Requires q_per_idx >= 1 and
 *   0 <= q_pos0, q_pos0 + n_q <= n_kv.
 */
DSA_API int sparse_attn_topk_shared(const void* Q, const void* K, const void* V, const int32_t* idx,
                            int B, int n_q, int q_pos0, int n_kv, int Hq, int Hkv, int d_qk, int d_v,
                            int topk, int q_per_idx, float scale, void* O, int o_dtype,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ======================================================================
 * Paged, variable-length decode (serving).
 *
 * The same decode-step operations ([QbitAI] §IndexCache: the indexer picks
 * each new token's important history tokens; [Explainer] §稀疏注意力: the
 * attention reads only those) over a batch of sequences of different
 * lengths whose caches live in a shared pool of fixed-size pages.  Token t
 * of sequence b is row page_table[b * max_pages + t / page_size] *
 * page_size + t % page_size of the pool; seq_lens[b] counts its cached
 * tokens, the new token (the query) being the last of them.
 *
 * idx_score_topk_paged: one query per sequence.
 *   q_I        [B, H_I, d_I] bf16        w [B, H_I] fp32
 *   k_pages    [num_pages * page_size, d_I] bf16
 *   page_table [B, max_pages] int32 (device), seq_lens [B] int32 (device)
 *   idx_out    [B, topk] int32: logical token indices, ascending, then -1.
 * Requires H_I in {32, 64}, d_I = 128, page_size a power of two >= 16,
 * max_pages * page_size >= max_seq_len >= every seq_lens[b] >= 1 (a length
 * outside [1, max_seq_len] is flagged DSA_STATUS_BAD_INDEX and clamped; page
 * numbers outside [0, num_pages) read page 0, whose keys are masked).
 * max_seq_len (host) sizes the work split and the per-sequence score keys
 * the selection reads (4 bytes per token of max_seq_len in the workspace).
 *
 * sparse_attn_topk_paged: attention of each sequence's query over its
 * selected tokens (logical indices, as idx_score_topk_paged writes them).
 *   Q [B, Hq, d] bf16; K_pages, V_pages [num_pages * page_size, Hkv, d]
 *   bf16; idx [B, topk]; O [B, Hq, d] fp32 or bf16.  d in {64, 128},
 *   Hq/Hkv <= 8.  Indices >= seq_lens[b] or mapping to a page outside
 *   [0, num_pages) are skipped and flagged.  Workspace:
 *   sparse_attn_topk_workspace_size(B, 1, num_pages * page_size, ...).
 *
 * sparse_attn_topk_paged_e4m3: the same attention over a K/V cache kept
 *   as OCP E4M3 codes (1 byte each, bias 7, max 448) with one fp32 scale
 *   per (token, KV head): the real K row is code x k_scale, likewise V.
 *   K8_pages, V8_pages [num_pages * page_size, Hkv, d] uint8 codes;
 *   k_scale, v_scale [num_pages * page_size, Hkv] fp32; Q bf16 as above.
 *   Arithmetic: Q is taken to fp16, K codes widen exactly to fp16 and the
 *   K scale multiplies the fp32 score; V rows are code x scale rounded to
 *   fp16; fp32 accumulation and softmax.  Same shapes, rules, flags and
 *   workspace as sparse_attn_topk_paged.  The gather reads half the bytes
 *   of a bf16 cache, which is what bounds decode attention.
 * ====================================================================== */
DSA_API int idx_score_topk_paged_workspace_size(int B, int max_seq_len, int H_I, int d_I, int topk,
                                                size_t* bytes);
DSA_API int idx_score_topk_paged(const void* q_I, const void* k_pages, const int32_t* page_table,
                                 const int32_t* seq_lens, const float* w, int B, int max_seq_len,
                                 int page_size, int num_pages, int max_pages, int H_I, int d_I, int topk,
                                 int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream);
DSA_API int sparse_attn_topk_paged(const void* Q, const void* K_pages, const void* V_pages,
                                   const int32_t* page_table, const int32_t* seq_lens, const int32_t* idx,
                                   int B, int page_size, int num_pages, int max_pages, int Hq, int Hkv,
                                   int d, int topk, float scale, void* O, int o_dtype,
                                   void* workspace, size_t workspace_bytes, void* stream);
DSA_API int sparse_attn_topk_paged_e4m3(const void* Q, const void* K8_pages, const float* k_scale,
                                        const void* V8_pages, const float* v_scale,
                                        const int32_t* page_table, const int32_t* seq_lens,
                                        const int32_t* idx, int B, int page_size, int num_pages,
                                        int max_pages, int Hq, int Hkv, int d, int topk, float scale,
                                        void* O, int o_dtype, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* ======================================================================
 * F/S pattern search -- which layers of a group keep their indexer.
 *
 * [QbitAI] §IndexCache: for an existing model, the layers worth keeping are
 * searched by the change in loss; [Explainer] §训练无关: a greedy pass over a
 * small calibration batch picks the F and S layers, weights untouched.  The
 * loss proxy here is selection overlap (the pages report 70-100% between
 * adjacent layers): an S layer reusing F layer f's top-k loses the part of
 * its own top-k that f's misses.  Steps: run every layer as F on calibration
 * rows (idx_score_topk), measure overlaps (idx_overlap), search
 * (layer_pattern_search), then run groups with the pattern found.
 * ====================================================================== */

/* counts[r] = |A_r ∩ B_r| for rows r of two [rows, topk] int32 index buffers
 * in the canonical layout (ascending indices, then -1; as idx_score_topk
 * writes them).  Device pointers; asynchronous on `stream`.  Rows out of the
 * canonical layout give unspecified counts (never out-of-bounds reads). */
DSA_API int idx_overlap(const int32_t* idx_a, const int32_t* idx_b, int64_t rows, int topk,
                        int32_t* counts, void* stream);

/* Greedy removal from the all-F pattern.  overlap: host [n_layers][n_layers]
 * doubles, row-major, overlap[f][j] (f < j, in [0,1]) = mean fraction of
 * layer j's selection that layer f's selection also holds; other entries are
 * not read.  Loss of a pattern = sum over its S layers j of
 * (1 - overlap[f][j]), f the most recent F layer before j.  While more than
 * n_f layers are F, the F layer (never layer 0) whose turning into S gives the
 * smallest loss becomes S (the lowest such layer on ties).  Writes n_layers
 * characters 'F'/'S' and a terminating NUL to host pattern_out. */
DSA_API int layer_pattern_search(const double* overlap, int n_layers, int n_f, char* pattern_out);

/* ======================================================================
 * layer_group_forward -- one layer group: F layers index, S layers reuse.
 *
 * [QbitAI] §IndexCache: few layers keep an indexer, compute the top-k and
 * cache it, the rest skip it and reuse the most recent result with one
 * extra branch in the inference code; §GLM-5.2 and [Explainer] §sharing:
 * groups of four, the first layer computes.  `pattern` is a string over
 * {F, S} of length n_layers starting with F (e.g. "FSSS", "FSSSFSSS").
 * For each layer l in order: if pattern[l]=='F', idx_score_topk writes
 * the cache buffer; then sparse_attn_topk runs with layer l's own Q/K/V
 * and the cached indices.  S layers launch no indexer work.
 * ====================================================================== */
typedef struct dsa_group_shape {
    int B, n_q, q_pos0, n_kv;
    int H_I, d_I, idx_dtype;      /* indexer (DSA_BF16 or DSA_E4M3) */
    int Hq, Hkv, d_qk, d_v;       /* attention                      */
    int topk;
    float scale;                  /* <= 0 selects 1/sqrt(d_qk)      */
    int o_dtype;                  /* DSA_F32 or DSA_BF16            */
} dsa_group_shape;

typedef struct dsa_layer_args {
    /* indexer inputs, read on F layers only (may be NULL on S layers) */
    const void* q_I; const float* q_scale; const void* k_I; const float* k_scale; const float* w;
    /* attention inputs and output of this layer */
    const void* Q; const void* K; const void* V; void* O;
} dsa_layer_args;

typedef struct dsa_group_stats {
    int indexer_launches;     /* idx_score_topk calls made           */
    int attention_launches;   /* sparse_attn_topk calls made         */
    /* Optional per-layer timing.  If non-NULL, `events` holds 3*n_layers
     * cudaEvent_t handles (as void*) owned by the caller; on `stream` the
     * library records events[3l] before layer l's indexer launch,
     * events[3l+1] after it (same point on S layers) and events[3l+2]
     * after layer l's attention launch. */
    void* const* events;
} dsa_group_stats;

DSA_API int layer_group_forward_workspace_size(const dsa_group_shape* shape, size_t* bytes);
DSA_API int layer_group_forward(const dsa_group_shape* shape, const dsa_layer_args* layers, int n_layers,
                        const char* pattern, dsa_index_cache* cache, dsa_group_stats* stats,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ======================================================================
 * idx_score_topk_noalloc -- idx_score_topk for callers that cannot
 * allocate device memory.  (The pages have no counterpart: this is a
 * deployment variant of the same fused indexer + top-k.)
 *
 * Who needs it: code that runs inside another runtime's memory pool (an
 * inference server or graph executor that owns every device allocation and
 * forbids cudaMalloc, which can also synchronise the whole device), or a
 * latency-critical path that must not allocate.  Such callers cannot
 * provide the workspace idx_score_topk asks for.  This entry point takes
 * only the inputs and the output (same meaning and layout as
 * idx_score_topk) and keeps its scratch in one fixed 32 MiB array inside
 * the library; it calls no allocator.
 *   - The array is held by every GPU that loads the library until exit.
 *   - The kernel's grid is capped to the CTAs whose top-k candidate buffers
 *     fit in the array (63 at H_I = 32, topk = 2048), so big problems run
 *     more slowly than with a full workspace.  A problem whose single CTA
 *     needs more than the array is rejected with DSA_ERR_UNSUPPORTED.
 *   - All calls share the array and it keeps the last call's contents;
 *     each call clears the part that must start at zero.  Calls that
 *     overlap on the GPU race on it and must be serialised by the caller.
 *   - The first call on each device resolves the array's address
 *     (cudaGetSymbolAddress); make that first call before any stream
 *     capture begins.
 *   - Device-side status (timeouts) is not reported by this entry point.
 * ====================================================================== */
DSA_API int idx_score_topk_noalloc(const void* q_I, const float* q_scale, const void* k_I,
                                   const float* k_scale, const float* w, int dtype, int B, int n_q,
                                   int q_pos0, int n_kv, int H_I, int d_I, int topk,
                                   int32_t* idx_out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
