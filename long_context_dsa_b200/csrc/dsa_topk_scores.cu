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

// ---------------------------------------------------------------------------
// Bitmap merge: the final top-k of a row from its `len` (key, token) pairs when the
// tokens are distinct and below n_tok (the split decode indexer's partial lists).
// One 512-thread CTA per row reads the pairs from L2: a radix select over the keys
// (8-bit digits from the highest bit where they differ) finds the k-th key, a second
// one over the tokens settles ties at it (lower tokens first); the survivors then set
// their token's bit in a bitmap of the row's positions, which is read back in order.
// ---------------------------------------------------------------------------
static constexpr int kMbThreads = 512, kMbWarps = kMbThreads / 32;

struct MergeScratch {
    int hist[kMbWarps][256];
    int warp_val[kMbWarps];
    int sel_digit, sel_above, sel_equal;
};

// kk-th largest (1-based) value among the items `want` accepts, value = get(i).
template <class Get, class Want>
__device__ uint32_t block_kth(MergeScratch* sc, int n, int kk, Get get, Want want, int& n_above, int& n_equal) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    // range of the participating values
    uint32_t hi = 0u, lo_inv = 0u;
    for (int i = tid; i < n; i += kMbThreads)
        if (want(i)) {
            const uint32_t v = get(i);
            hi = max(hi, v);
            lo_inv = max(lo_inv, ~v);
        }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        lo_inv = max(lo_inv, __shfl_xor_sync(0xffffffffu, lo_inv, off));
    }
    if (lane == 0) {
        sc->hist[w][0] = static_cast<int>(hi);
        sc->hist[w][1] = static_cast<int>(lo_inv);
    }
    __syncthreads();
    hi = 0u;
    lo_inv = 0u;
    for (int j = 0; j < kMbWarps; ++j) {
        hi = max(hi, static_cast<uint32_t>(sc->hist[j][0]));
        lo_inv = max(lo_inv, static_cast<uint32_t>(sc->hist[j][1]));
    }
    __syncthreads();
    const uint32_t diff = hi ^ ~lo_inv;
    int nbits = diff ? 32 - __clz(diff) : 0;
    uint32_t fixed = nbits >= 32 ? 0u : ~((1u << nbits) - 1u);
    uint32_t prefix = hi & fixed;
    int above = 0, equal = 0;
    if (nbits == 0) {  // every participant equal: count them
        int c = 0;
        for (int i = tid; i < n; i += kMbThreads) c += want(i) ? 1 : 0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
        if (lane == 0) sc->warp_val[w] = c;
        __syncthreads();
        for (int j = 0; j < kMbWarps; ++j) equal += sc->warp_val[j];
        __syncthreads();
    }
    while (nbits > 0) {
        const int width = nbits < 8 ? nbits : 8;
        const int shift = nbits - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int b = tid; b < kMbWarps * 256; b += kMbThreads) (&sc->hist[0][0])[b] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kMbThreads)
            if (want(i)) {
                const uint32_t v = get(i);
                if ((v & fixed) == prefix) atomicAdd(&sc->hist[w][(v >> shift) & dmask], 1);
            }
        __syncthreads();
        if (w == 0) {
            int cnt8[8], s8 = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                int c = 0;
                for (int ww = 0; ww < kMbWarps; ++ww) c += sc->hist[ww][lane * 8 + j];
                cnt8[j] = c;
                s8 += c;
            }
            int suf = s8;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_down_sync(0xffffffffu, suf, off);
                if (lane + off < 32) suf += o;
            }
            const unsigned ball = __ballot_sync(0xffffffffu, suf >= kk);
            const int L = 31 - __clz(ball);
            if (lane == L) {
                int acc = suf - s8;
                bool found = false;
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    if (!found && acc + cnt8[j] >= kk) {
                        sc->sel_digit = L * 8 + j;
                        sc->sel_above = acc;
                        sc->sel_equal = cnt8[j];
                        found = true;
                    }
                    acc += cnt8[j];
                }
            }
        }
        __syncthreads();
        kk -= sc->sel_above;
        above += sc->sel_above;
        equal = sc->sel_equal;
        prefix |= static_cast<uint32_t>(sc->sel_digit) << shift;
        fixed |= dmask << shift;
        nbits = shift;
        __syncthreads();
    }
    n_above = above;
    n_equal = equal;
    return prefix;
}

__global__ void __launch_bounds__(kMbThreads, 1)
    topk_merge_bitmap_kernel(const uint32_t* __restrict__ keys, const int* __restrict__ idxs, int rows, int len,
                             int n_tok, int k, int* __restrict__ out, WsHeader* hdr) {
    extern __shared__ __align__(16) unsigned char smem[];
    MergeScratch* sc = reinterpret_cast<MergeScratch*>(smem);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + sizeof(MergeScratch));
    const int nw = (n_tok + 31) / 32;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const uint32_t* rk = keys + static_cast<size_t>(row) * len;
        const int* ri = idxs + static_cast<size_t>(row) * len;
        auto valid = [&](int i) {
            const int t = __ldg(ri + i);
            return t >= 0 && t < n_tok;
        };
        // survivors: keys above kstar, and keys equal to it with a token up to ithr
        int n_valid = 0;
        {
            int c = 0;
            for (int i = tid; i < len; i += kMbThreads) {
                const int t = __ldg(ri + i);
                if (t >= n_tok) raise_status(hdr, DSA_STATUS_BAD_INDEX, t);
                c += (t >= 0 && t < n_tok) ? 1 : 0;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
            if (lane == 0) sc->warp_val[w] = c;
            __syncthreads();
            for (int j = 0; j < kMbWarps; ++j) n_valid += sc->warp_val[j];
            __syncthreads();
        }
        uint32_t kstar = 0u, ithr = 0xffffffffu;
        const bool keep_all = n_valid <= k;
        if (!keep_all) {
            int G, E;
            kstar = block_kth(sc, len, k, [&](int i) { return __ldg(rk + i); }, valid, G, E);
            const int kk = k - G;
            if (E > kk) {
                int g2, e2;
                ithr = ~block_kth(sc, len, kk, [&](int i) { return ~static_cast<uint32_t>(__ldg(ri + i)); },
                                  [&](int i) { return valid(i) && __ldg(rk + i) == kstar; }, g2, e2);
            }
        }
        for (int j = tid; j < nw; j += kMbThreads) bits[j] = 0u;
        __syncthreads();
        for (int i = tid; i < len; i += kMbThreads) {
            if (!valid(i)) continue;
            const uint32_t key = __ldg(rk + i);
            const int t = __ldg(ri + i);
            const bool keep = keep_all || key > kstar || (key == kstar && static_cast<uint32_t>(t) <= ithr);
            if (keep) atomicOr(&bits[t >> 5], 1u << (t & 31));
        }
        __syncthreads();
        // read the bitmap back in order: each thread a contiguous run of words
        const int per = (nw + kMbThreads - 1) / kMbThreads;
        const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
        int c = 0;
        for (int j = w0; j < w1; ++j) c += __popc(bits[j]);
        int inc = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) sc->warp_val[w] = inc;
        __syncthreads();
        int base = inc - c;
        for (int j = 0; j < w; ++j) base += sc->warp_val[j];
        int* orow = out + static_cast<size_t>(row) * k;
        for (int j = w0; j < w1; ++j) {
            uint32_t m = bits[j];
            while (m) {
                const int b = __ffs(m) - 1;
                if (base < k) orow[base] = j * 32 + b;
                ++base;
                m &= m - 1u;
            }
        }
        const int total = min(n_valid, k);
        for (int j = total + tid; j < k; j += kMbThreads) orow[j] = -1;
        __syncthreads();
    }
}

// Final top-k of each row from `len` (key, token) pairs in ascending token order
// (the partial lists of the split decode indexer, -1 tokens skipped; tokens < n_tok).
cudaError_t launch_topk_merge_pairs(const uint32_t* keys, const int* idxs, int rows, int len, int k, int* out,
                                    WsHeader* hdr, int num_sms, cudaStream_t stream, int n_tok) {
    const size_t bitmap = static_cast<size_t>((n_tok + 31) / 32) * 4;
    if (n_tok > 0 && sizeof(MergeScratch) + bitmap <= 200 * 1024) {
        const size_t smem = sizeof(MergeScratch) + bitmap;
        cudaError_t e = cudaFuncSetAttribute(topk_merge_bitmap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        const int grid = rows < num_sms ? rows : num_sms;
        topk_merge_bitmap_kernel<<<grid, kMbThreads, smem, stream>>>(keys, idxs, rows, len, n_tok, k, out, hdr);
        return cudaGetLastError();
    }
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
