// dsa_topk_scores.cu -- the per-row top-k alone, on a given fp32 score array.
//
// The same selection rule and building blocks (dsa_topk.cuh) as the fused
// indexer, pruning with the exact radix select only; exists so a selection
// can be checked bit for bit against a reference on a given score array.  One 128-thread CTA owns a row at a time;
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

// One dense fp32 score row (entry j is token j) at a time per CTA; each warp meets its entries in
// ascending token order, as the selection code requires.
__global__ void __launch_bounds__(kTsThreads) topk_stream_kernel(const float* __restrict__ scores, int rows,
                                                                 int q_pos0, int n_kv, long long ld, int k,
                                                                 int* __restrict__ out, WsHeader* hdr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TopkScoresSmem& sm = *reinterpret_cast<TopkScoresSmem*>(smem_raw);
    TopkGroup<kTsThreads> grp{static_cast<int>(threadIdx.x), 1, &sm.scratch, kCandCap};
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int sub = grp.sub();
    uint32_t* wkey = sm.ckey + w * sub;  // this warp's sub-buffer
    int* widx = sm.cidx + w * sub;

    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int n = min(q_pos0 + r + 1, n_kv);
        int* orow = out + static_cast<long long>(r) * k;
        if (n <= k) {
            for (int j = tid; j < k; j += kTsThreads) orow[j] = (j < n) ? j : -1;
            continue;
        }
        if (tid == 0) topk_row_init(&sm.st);
        grp.sync();
        const float* srow = scores + static_cast<long long>(r) * ld;
        int nan_seen = 0;
        int cnt = 0;  // this warp's sub-buffer count (warp-uniform)
        for (int base = 0; base < n; base += kTsPerIter) {
            const uint32_t tk = sm.st.thr_key;
            const int ti = sm.st.thr_idx;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = base + i * kTsThreads + tid;
                const bool inb = j < n;
                const float s = inb ? __ldg(srow + j) : 0.f;
                nan_seen |= (inb && s != s);
                const uint32_t key = score_key(s);
                const int idx = j;
                const bool live = inb && s == s;
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
    cudaError_t e = cudaFuncSetAttribute(topk_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int per_sm = static_cast<int>((227 * 1024) / (smem + 1024));
    int grid = num_sms * (per_sm > 0 ? per_sm : 1);
    if (grid > rows) grid = rows;
    if (grid < 1) grid = 1;
    topk_stream_kernel<<<grid, kTsThreads, smem, stream>>>(scores, rows, q_pos0, n_kv, ld, k, out, hdr);
    return cudaGetLastError();
}

}  // namespace dsa
