// dsa_topk_scores.cu -- the per-row top-k alone, on a given fp32 score array.
//
// Same selection code (dsa_topk.cuh) and rule as the fused indexer; exists
// so the selection can be checked bit for bit against a reference that
// scores rows independently.  One 128-thread CTA owns a row at a time;
// the candidate buffer lives in the CTA's shared memory.
#include "dsa_topk.cuh"

namespace dsa {

static constexpr int kTsThreads = 128;
static constexpr int kTsPerIter = kTsThreads * 4;  // scores read per step

struct TopkScoresSmem {
    uint32_t ckey[kCandCap];
    int cidx[kCandCap];
    int sortbuf[DSA_TOPK_MAX];
    TopkGroup<kTsThreads>::Scratch scratch;
    TopkRowState st;
};

// One row at a time per CTA.  Input is either a dense fp32 score row
// (PAIRS = false: entry j is token j) or a list of (score key, token) pairs
// in ascending token order with -1 tokens skipped (PAIRS = true: merging
// partial top-k lists).  Either way each warp meets its entries in
// ascending token order, as the selection code requires.
template <bool PAIRS>
__global__ void __launch_bounds__(kTsThreads) topk_stream_kernel(const float* __restrict__ scores,
                                                                 const uint32_t* __restrict__ pkeys,
                                                                 const int* __restrict__ pidx, int rows, int q_pos0,
                                                                 int n_kv, long long ld, int k,
                                                                 int* __restrict__ out, WsHeader* hdr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TopkScoresSmem& sm = *reinterpret_cast<TopkScoresSmem*>(smem_raw);
    TopkGroup<kTsThreads> grp{static_cast<int>(threadIdx.x), 1, &sm.scratch, kCandCap};
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int sub = grp.sub();
    uint32_t* wkey = sm.ckey + w * sub;  // this warp's sub-buffer
    int* widx = sm.cidx + w * sub;

    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        // PAIRS: n_kv is the list length; every entry is a candidate
        const int n = PAIRS ? n_kv : min(q_pos0 + r + 1, n_kv);
        int* orow = out + static_cast<long long>(r) * k;
        if (!PAIRS && n <= k) {
            for (int j = tid; j < k; j += kTsThreads) orow[j] = (j < n) ? j : -1;
            continue;
        }
        if (tid == 0) topk_row_init(&sm.st);
        grp.sync();
        const float* srow = scores + static_cast<long long>(r) * ld;
        const uint32_t* krow = pkeys + static_cast<long long>(r) * ld;
        const int* irow = pidx + static_cast<long long>(r) * ld;
        int nan_seen = 0;
        int cnt = 0;  // this warp's sub-buffer count (warp-uniform)
        for (int base = 0; base < n; base += kTsPerIter) {
            const uint32_t tk = sm.st.thr_key;
            const int ti = sm.st.thr_idx;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = base + i * kTsThreads + tid;
                const bool inb = j < n;
                uint32_t key;
                int idx;
                bool live;
                if (PAIRS) {
                    idx = inb ? __ldg(irow + j) : -1;
                    key = inb ? __ldg(krow + j) : 0u;
                    live = idx >= 0;
                } else {
                    const float s = inb ? __ldg(srow + j) : 0.f;
                    nan_seen |= (inb && s != s);
                    key = score_key(s);
                    idx = j;
                    live = inb && s == s;
                }
                const bool adm = live & ((key > tk) | ((key == tk) & (idx < ti)));
                topk_append_warp(wkey, widx, cnt, key, idx, adm, sub);
            }
            if (lane == 0) sm.st.cnt[w] = cnt;
            if (cnt > sub && lane == 0) raise_status(hdr, DSA_STATUS_OVERFLOW, cnt);
            grp.sync();
            int mx = 0, tot = 0;
#pragma unroll
            for (int ww = 0; ww < 4; ++ww) {
                mx = max(mx, sm.st.cnt[ww]);
                tot += sm.st.cnt[ww];
            }
            grp.sync();  // every thread has read the counts before any is rewritten
            if (mx > sub - kTsPerIter / 4 && tot > k) {
                grp.prune(&sm.st, sm.ckey, sm.cidx, k, sub - kTsPerIter / 4 - 32, sm.sortbuf);
                cnt = sm.st.cnt[w];
            }
        }
        if (nan_seen) raise_status(hdr, DSA_STATUS_NAN_SCORE, r);
        if (lane == 0) sm.st.cnt[w] = cnt;
        grp.sync();
        grp.finish(&sm.st, sm.ckey, sm.cidx, k, orow, nullptr, sm.sortbuf);
    }
}

size_t topk_scores_smem_bytes() { return sizeof(TopkScoresSmem); }

cudaError_t launch_topk_scores(const float* scores, int rows, int q_pos0, int n_kv, long long ld, int k,
                               int* out, WsHeader* hdr, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(TopkScoresSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_stream_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int per_sm = static_cast<int>((227 * 1024) / (smem + 1024));
    int grid = num_sms * (per_sm > 0 ? per_sm : 1);
    if (grid > rows) grid = rows;
    if (grid < 1) grid = 1;
    topk_stream_kernel<false><<<grid, kTsThreads, smem, stream>>>(scores, nullptr, nullptr, rows, q_pos0, n_kv, ld, k,
                                                                 out, hdr);
    return cudaGetLastError();
}

// Final top-k of each row from `len` (key, token) pairs in ascending token order
// (the partial lists of the split decode indexer, -1 tokens skipped).
cudaError_t launch_topk_merge_pairs(const uint32_t* keys, const int* idxs, int rows, int len, int k, int* out,
                                    WsHeader* hdr, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(TopkScoresSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_stream_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int grid = rows < num_sms * 4 ? rows : num_sms * 4;
    if (grid < 1) grid = 1;
    topk_stream_kernel<true><<<grid, kTsThreads, smem, stream>>>(nullptr, keys, idxs, rows, 0, len, len, k, out, hdr);
    return cudaGetLastError();
}

}  // namespace dsa
