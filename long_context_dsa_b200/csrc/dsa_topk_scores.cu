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
    TopkScratch scratch;
    TopkRowState st;
};

__global__ void __launch_bounds__(kTsThreads) topk_scores_kernel(const float* __restrict__ scores, int rows,
                                                                 int q_pos0, int n_kv, long long ld, int k,
                                                                 int* __restrict__ out, WsHeader* hdr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TopkScoresSmem& sm = *reinterpret_cast<TopkScoresSmem*>(smem_raw);
    TopkGroup<kTsThreads> grp{static_cast<int>(threadIdx.x), 1, &sm.scratch, kCandCap};
    const int tid = threadIdx.x;

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
        for (int base = 0; base < n; base += kTsPerIter) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = base + i * kTsThreads + tid;
                const bool inb = j < n;
                const float s = inb ? __ldg(srow + j) : 0.f;
                nan_seen |= (inb && s != s);
                const uint32_t key = score_key(s);
                const bool adm = inb && topk_admit(&sm.st, key, j);
                topk_append_warp(&sm.st, sm.ckey, sm.cidx, key, j, adm, kCandCap, hdr);
            }
            grp.sync();
            const int c = sm.st.count;  // read by every thread before anyone appends again
            grp.sync();
            if (c > kCandCap - kTsPerIter) grp.prune(&sm.st, sm.ckey, sm.cidx, k);
        }
        if (nan_seen) raise_status(hdr, DSA_STATUS_NAN_SCORE, r);
        grp.finish(&sm.st, sm.ckey, sm.cidx, k, orow, sm.sortbuf);
    }
}

size_t topk_scores_smem_bytes() { return sizeof(TopkScoresSmem); }

cudaError_t launch_topk_scores(const float* scores, int rows, int q_pos0, int n_kv, long long ld, int k,
                               int* out, WsHeader* hdr, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(TopkScoresSmem);
    cudaError_t e = cudaFuncSetAttribute(topk_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int per_sm = static_cast<int>((227 * 1024) / (smem + 1024));
    int grid = num_sms * (per_sm > 0 ? per_sm : 1);
    if (grid > rows) grid = rows;
    if (grid < 1) grid = 1;
    topk_scores_kernel<<<grid, kTsThreads, smem, stream>>>(scores, rows, q_pos0, n_kv, ld, k, out, hdr);
    return cudaGetLastError();
}

}  // namespace dsa
