// dsa_topk_radix.cu -- per-row top-k of a few long rows of score keys, spread over many CTAs.
//
// Same selection rule as every other top-k in the library ([Term] "dot product + top-k"; ties
// to the lower token index, output ascending then -1): for a decode step the one-query indexer
// writes its row of order-preserving score keys (4 bytes per cached token: 4 MB at a 1M-token
// cache, against the 134 MB of fp8 keys it reads), and the selection runs here as a radix
// select over all the row's keys, with every SM taking a slice:
//   * 4 histogram passes of 8 bits each, from the top bit down.  Each CTA counts the keys of its
//     slice that match the prefix found so far (shared-memory histogram, then global atomics);
//     the last CTA of the row to finish (atomic ticket, no waiting) picks the digit holding the
//     k-th key, extends the prefix and clears the histogram for the next pass.  After 4 passes
//     the prefix is the k-th largest key K and `kk` says how many keys equal to K are selected.
//   * A count pass: keys above K and keys equal to K in each slice.
//   * A write pass: each CTA places its selected tokens (keys above K, and the first kk keys
//     equal to K in token order) at their rank among the row's selections -- slices are token
//     ranges in order, so the output is ascending -- and pads the row with -1.
// No CTA ever waits for another: the passes are separate launches.
#include "dsa_common.cuh"

namespace dsa {

namespace {

constexpr int kRxThreads = 256;
constexpr int kRxBins = 256;  // 8-bit digits (wider digits cost more in histogram clears and
                               // flushes than the pass they save: measured with 3 x 11 bits)
constexpr int kRxPasses = 4;
// pass p covers bits [shift, shift + 8) of the key
__host__ __device__ constexpr int rx_shift(int pass) { return 24 - 8 * pass; }
__host__ __device__ constexpr int rx_width(int pass) { return 8 + 0 * pass; }

struct RadixRow {
    uint32_t prefix;  // the k-th key's bits found so far
    int kk;           // how many of the keys matching the prefix are still to select
    int ticket;       // CTAs of the row done with the current pass
    int pad;
};

__global__ void __launch_bounds__(kRxThreads)
    radix_init_kernel(RadixRow* rs, int* hist, int rows, int k) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * kRxBins; i += gridDim.x * blockDim.x) hist[i] = 0;
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x) {
        rs[r].prefix = 0u;
        rs[r].kk = k;
        rs[r].ticket = 0;
        rs[r].pad = 0;
    }
}

// Pass `pass` (0 = bits 31..24): histogram of the next digit of the keys that match the prefix.
__global__ void __launch_bounds__(kRxThreads)
    radix_hist_kernel(const uint32_t* __restrict__ keys, long long ld, int n, int nblk, int per, int pass, int k,
                      RadixRow* rs, int* hist) {
    __shared__ int sh[kRxBins];
    __shared__ int last;
    const int row = blockIdx.x / nblk, blk = blockIdx.x % nblk;
    const int shift = rx_shift(pass);
    const uint32_t dmask = (1u << rx_width(pass)) - 1u;
    const uint32_t fixed = pass == 0 ? 0u : (0xffffffffu << (shift + rx_width(pass)));
    const uint32_t prefix = rs[row].prefix;
    const int kk = rs[row].kk;
    for (int b = threadIdx.x; b < kRxBins; b += kRxThreads) sh[b] = 0;
    __syncthreads();
    if (n > k) {  // (rows no longer than k select everything; nothing to count)
        const uint32_t* kr = keys + row * ld;
        const int i0 = blk * per, i1 = min(n, i0 + per);
        // the keys of a row share their top bits, so most lanes of a warp hit the same bin:
        // one shared-memory atomic per distinct digit per warp.  Keys are read kBatch at a time
        // into registers first, so the loads overlap instead of waiting behind each vote.
        constexpr int kBatch = 8;
        for (int c0 = i0; c0 < i1; c0 += kRxThreads * kBatch) {
            uint32_t kv[kBatch];
#pragma unroll
            for (int e = 0; e < kBatch; ++e) {
                const int i = c0 + e * kRxThreads + threadIdx.x;
                kv[e] = i < i1 ? __ldg(kr + i) : 0u;
            }
#pragma unroll
            for (int e = 0; e < kBatch; ++e) {
                const int i = c0 + e * kRxThreads + threadIdx.x;
                const bool in = i < i1 && (kv[e] & fixed) == prefix;
                const unsigned active = __ballot_sync(0xffffffffu, in);
                if (in) {
                    const uint32_t dg = (kv[e] >> shift) & dmask;
                    const unsigned same = __match_any_sync(active, dg);
                    if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&sh[dg], __popc(same));
                }
            }
        }
    }
    __syncthreads();
    int* hr = hist + row * kRxBins;
    for (int b = threadIdx.x; b < kRxBins; b += kRxThreads)
        if (sh[b]) atomicAdd(hr + b, sh[b]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = (atomicAdd(&rs[row].ticket, 1) == nblk - 1);
    __syncthreads();
    if (!last) return;
    // the row's last CTA: every other CTA's counts are in (they fenced before taking a ticket)
    __threadfence();
    if (threadIdx.x < 32) {
        // lane l owns bins 8 l .. 8 l + 7; the digit holding the need-th largest key
        const int lane = threadIdx.x;
        constexpr int PB = kRxBins / 32;
        int s64 = 0;
        for (int j = 0; j < PB; ++j) s64 += atomicAdd(hr + lane * PB + j, 0);  // read through L2
        int suf = s64;  // keys in bins >= lane * PB
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_down_sync(0xffffffffu, suf, off);
            if (lane + off < 32) suf += o;
        }
        const int need = min(kk, n);
        const unsigned ball = __ballot_sync(0xffffffffu, suf >= need);
        const int L = ball ? 31 - __clz(ball) : 0;
        if (lane == L) {
            int acc = suf - s64;
            int d = 0, above = 0;
            for (int j = PB - 1; j >= 0; --j) {
                const int c = atomicAdd(hr + lane * PB + j, 0);
                if (acc + c >= need) {
                    d = lane * PB + j;
                    above = acc;
                    break;
                }
                acc += c;
            }
            rs[row].prefix = prefix | (static_cast<uint32_t>(d) << shift);
            rs[row].kk = need - above;
        }
        __syncwarp();
        for (int j = 0; j < PB; ++j) hr[lane * PB + j] = 0;
        if (lane == 0) rs[row].ticket = 0;
    }
}

// Keys above the k-th key and keys equal to it, per slice.
__global__ void __launch_bounds__(kRxThreads)
    radix_count_kernel(const uint32_t* __restrict__ keys, long long ld, int n, int nblk, int per, int k,
                       const RadixRow* rs, int2* counts) {
    __shared__ int wg[kRxThreads / 32], we[kRxThreads / 32];
    const int row = blockIdx.x / nblk, blk = blockIdx.x % nblk;
    const uint32_t K = rs[row].prefix;
    const uint32_t* kr = keys + row * ld;
    const int i0 = blk * per, i1 = min(n, i0 + per);
    int g = 0, e = 0;
    if (n > k)
        for (int i = i0 + threadIdx.x; i < i1; i += kRxThreads) {
            const uint32_t key = __ldg(kr + i);
            g += key > K;
            e += key == K;
        }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, off);
        e += __shfl_xor_sync(0xffffffffu, e, off);
    }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        wg[w] = g;
        we[w] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int tg = 0, te = 0;
        for (int j = 0; j < kRxThreads / 32; ++j) {
            tg += wg[j];
            te += we[j];
        }
        counts[blockIdx.x] = make_int2(tg, te);
    }
}

// Selected tokens of each slice, at their rank among the row's selections; -1 after the last.
// Each thread takes a contiguous run of the slice: it counts its keys above K and equal to K, one
// block-wide scan gives every thread its rank among the equal keys and among the selections,
// then the thread writes its selected tokens in order.
__device__ __forceinline__ int2 block_excl_scan2(int2 v, int2* warp_tot, int2* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int2 inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int ox = __shfl_up_sync(0xffffffffu, inc.x, off), oy = __shfl_up_sync(0xffffffffu, inc.y, off);
        if (lane >= off) {
            inc.x += ox;
            inc.y += oy;
        }
    }
    if (lane == 31) warp_tot[w] = inc;
    __syncthreads();
    int2 before = make_int2(0, 0), tot = make_int2(0, 0);
#pragma unroll
    for (int j = 0; j < kRxThreads / 32; ++j) {
        const int2 t = warp_tot[j];
        if (j < w) {
            before.x += t.x;
            before.y += t.y;
        }
        tot.x += t.x;
        tot.y += t.y;
    }
    __syncthreads();
    *total = tot;
    return make_int2(before.x + inc.x - v.x, before.y + inc.y - v.y);
}

__global__ void __launch_bounds__(kRxThreads)
    radix_write_kernel(const uint32_t* __restrict__ keys, long long ld, int n, int nblk, int per, int k,
                       const RadixRow* rs, const int2* counts, int* __restrict__ out) {
    __shared__ int2 wt[kRxThreads / 32];
    __shared__ int base_out, base_eq;
    const int row = blockIdx.x / nblk, blk = blockIdx.x % nblk;
    int* orow = out + static_cast<long long>(row) * k;
    const int i0 = blk * per, i1 = min(n, i0 + per);
    if (n <= k) {  // every token of the row, then padding
        for (int i = i0 + threadIdx.x; i < i1; i += kRxThreads) orow[i] = i;
        if (blk == nblk - 1)
            for (int j = n + threadIdx.x; j < k; j += kRxThreads) orow[j] = -1;
        return;
    }
    const uint32_t K = rs[row].prefix;
    const int kk = rs[row].kk;  // keys equal to K to take, lowest tokens first
    {
        // keys above K and keys equal to K in the slices before this one
        int2 c = make_int2(0, 0);
        for (int j = threadIdx.x; j < blk; j += kRxThreads) {
            const int2 x = counts[row * nblk + j];
            c.x += x.x;
            c.y += x.y;
        }
        int2 tot;
        block_excl_scan2(c, wt, &tot);
        if (threadIdx.x == 0) {
            base_out = tot.x + min(tot.y, kk);  // equal keys are taken in token order
            base_eq = tot.y;
        }
        __syncthreads();
    }
    const uint32_t* kr = keys + row * ld;
    const int ipt = (per + kRxThreads - 1) / kRxThreads;  // this thread's run: [a, b)
    const int a = min(i1, i0 + threadIdx.x * ipt), b = min(i1, a + ipt);
    int2 mine = make_int2(0, 0);  // (above K, equal to K) in the run
    for (int i = a; i < b; ++i) {
        const uint32_t key = __ldg(kr + i);
        mine.x += key > K;
        mine.y += key == K;
    }
    int2 tot;
    const int2 pre = block_excl_scan2(mine, wt, &tot);  // within the slice
    int eq_rank = base_eq + pre.y;                        // equal keys before this run, row-wide
    // selections before this run: keys above K, plus the equal keys that made the cut
    int2 sel_mine = make_int2(mine.x + min(max(kk - eq_rank, 0), mine.y), 0);
    int2 tsel;
    int pos = base_out + block_excl_scan2(sel_mine, wt, &tsel).x;
    for (int i = a; i < b; ++i) {
        const uint32_t key = __ldg(kr + i);
        bool sel = key > K;
        if (key == K) {
            sel = eq_rank < kk;
            ++eq_rank;
        }
        if (sel) {
            if (pos < k) orow[pos] = i;
            ++pos;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Bin select: the same result for rows whose producer also counted their keys into a histogram of
// the top kBsBits bits (sign, 8 exponent bits, 4 mantissa bits of the score).
//   * compaction: every slice CTA finds the bin T holding its row's k-th largest key from the
//     histogram (suffix counts), then keeps its keys whose bin is >= T, in token order, in its own
//     region (at most kBsSliceCap) -- fewer than k keys above T plus the keys of bin T.
//   * final: one CTA per row loads the row's kept keys (at most kBsSmemCand) into shared memory in
//     token order, finds the k-th key K and how many keys equal to K to take by a radix select in
//     shared memory, and writes the selected tokens in order.  A row whose kept keys overflow
//     either bound (a score distribution packed into a few bins, many equal scores) is selected
//     by the same CTA directly from the full row instead.
constexpr int kBsBits = kBinTopkBits;
constexpr int kBsBins = 1 << kBsBits;
constexpr int kBsShift = 32 - kBsBits;
constexpr int kBsThreads = 512;
constexpr int kBsSliceCap = 2048;
constexpr int kBsSmemCand = 16384;

// The largest bin T with count(bins >= T) >= k in one row's histogram (0 when the row holds k
// keys or fewer: everything is kept); every thread of the kRxThreads-thread block gets it.
__device__ int bs_threshold_bin(const int* __restrict__ h, int k, int* hs, int* tsum, int* res) {
    constexpr int PB = kBsBins / kRxThreads;  // bins per thread
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    // the histogram into shared memory with coalesced 16-byte loads, then contiguous ranges per thread
    for (int i = t; i < kBsBins / 4; i += kRxThreads)
        reinterpret_cast<int4*>(hs)[i] = __ldg(reinterpret_cast<const int4*>(h) + i);
    __syncthreads();
    int v[PB];
    int s = 0;
#pragma unroll
    for (int j = 0; j < PB; ++j) {
        v[j] = hs[t * PB + ((j + t) & (PB - 1))];  // rotated start: no bank conflicts
        s += v[j];
    }
    // suffix sums over threads (thread t: keys in bins >= t * PB): warp suffix scan, then warps
    int suf = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += o;
    }
    if (lane == 0) tsum[w] = suf;  // this warp's total
    if (t == 0) *res = 0;
    __syncthreads();
    int later = 0;  // keys in the warps above this one
    for (int j = w + 1; j < kRxThreads / 32; ++j) later += tsum[j];
    suf += later;
    const int above_me = suf - s;
    if (suf >= k && above_me < k) {
        int acc = above_me, T = t * PB;
        for (int j = PB - 1; j >= 0; --j) {
            acc += hs[t * PB + j];
            if (acc >= k) {
                T = t * PB + j;
                break;
            }
        }
        *res = T;
    }
    __syncthreads();
    const int T = *res;
    __syncthreads();
    return T;
}

// Keys of one slice with bin >= T, in token order, into the slice's region; the slice's count
// (uncapped: a count above kBsSliceCap marks the row for the whole-row select).  Each thread
// takes 8 consecutive keys of a 2048-key chunk, a block scan orders the kept keys, and a running
// base carries across chunks.
__global__ void __launch_bounds__(kRxThreads)
    bin_compact_kernel(const uint32_t* __restrict__ keys, long long ld, int n, int nblk, int per, int k,
                       const int* __restrict__ hist, uint32_t* __restrict__ ckey, int* __restrict__ cidx,
                       int* __restrict__ ccnt) {
    __shared__ int2 wt[kRxThreads / 32];
    __shared__ int tsum[kRxThreads / 32];
    __shared__ int res;
    __shared__ __align__(16) int hs[kBsBins];
    const int row = blockIdx.x / nblk, blk = blockIdx.x % nblk;
    const uint32_t T = static_cast<uint32_t>(
        bs_threshold_bin(hist + static_cast<size_t>(row) * kBsBins, k, hs, tsum, &res));
    const uint32_t* kr = keys + row * ld;
    const int i0 = blk * per, i1 = min(n, i0 + per);
    uint32_t* ok = ckey + static_cast<size_t>(blockIdx.x) * kBsSliceCap;
    int* oi = cidx + static_cast<size_t>(blockIdx.x) * kBsSliceCap;
    int base = 0;
    for (int c0 = i0; c0 < i1; c0 += kRxThreads * 8) {
        const int a = c0 + threadIdx.x * 8;
        uint32_t kv[8];
        if (a + 8 <= i1 && ((row * ld + a) & 3) == 0) {
            const uint4 x = __ldg(reinterpret_cast<const uint4*>(kr + a));
            const uint4 y = __ldg(reinterpret_cast<const uint4*>(kr + a + 4));
            kv[0] = x.x; kv[1] = x.y; kv[2] = x.z; kv[3] = x.w;
            kv[4] = y.x; kv[5] = y.y; kv[6] = y.z; kv[7] = y.w;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) kv[e] = a + e < i1 ? __ldg(kr + a + e) : 0u;
        }
        int mine = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) mine += (a + e < i1) && (kv[e] >> kBsShift) >= T;
        int2 tot;
        int pos = base + block_excl_scan2(make_int2(mine, 0), wt, &tot).x;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if ((a + e < i1) && (kv[e] >> kBsShift) >= T) {
                if (pos < kBsSliceCap) {
                    ok[pos] = kv[e];
                    oi[pos] = a + e;
                }
                ++pos;
            }
        }
        base += tot.x;
    }
    if (threadIdx.x == 0) ccnt[blockIdx.x] = base;
}

// Block-wide exclusive scan of one int over kBsThreads threads (every thread gets its offset).
__device__ __forceinline__ int bs_excl_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) warp_tot[w] = inc;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int j = 0; j < kBsThreads / 32; ++j) {
        const int t = warp_tot[j];
        before += j < w ? t : 0;
        tot += t;
    }
    __syncthreads();
    *total = tot;
    return before + inc - v;
}

// The k-th largest of m keys produced by key_at(i) (i < m), and how many of the keys equal to it
// are selected; 4 passes of 8 bits with a shared-memory histogram.
template <class KeyAt>
__device__ void bs_kth(KeyAt key_at, int m, int k, int* sh, int* sel, uint32_t* K_out, int* kk_out) {
    uint32_t prefix = 0u;
    int need = min(k, m);
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        const uint32_t fixed = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
        for (int b = threadIdx.x; b < 256; b += kBsThreads) sh[b] = 0;
        __syncthreads();
        // the keys share their top bits, so most lanes of a warp hit the same bin: one shared
        // atomic per distinct digit per warp
        for (int i0 = 0; i0 < m; i0 += kBsThreads) {
            const int i = i0 + static_cast<int>(threadIdx.x);
            const uint32_t key = i < m ? key_at(i) : 0u;
            const bool in = i < m && (key & fixed) == prefix;
            const unsigned act = __ballot_sync(0xffffffffu, in);
            if (in) {
                const uint32_t dg = (key >> shift) & 255u;
                const unsigned same = __match_any_sync(act, dg);
                if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&sh[dg], __popc(same));
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int s8 = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) s8 += sh[lane * 8 + j];
            int suf = s8;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_down_sync(0xffffffffu, suf, off);
                if (lane + off < 32) suf += o;
            }
            const unsigned ball = __ballot_sync(0xffffffffu, suf >= need);
            const int L = ball ? 31 - __clz(ball) : 0;
            if (lane == L) {
                int acc = suf - s8, d = lane * 8;
                for (int j = 7; j >= 0; --j) {
                    const int c = sh[lane * 8 + j];
                    if (acc + c >= need) {
                        d = lane * 8 + j;
                        break;
                    }
                    acc += c;
                }
                sel[0] = static_cast<int>(prefix | (static_cast<uint32_t>(d) << shift));
                sel[1] = need - acc;
            }
        }
        __syncthreads();
        prefix = static_cast<uint32_t>(sel[0]);
        need = sel[1];
        __syncthreads();
    }
    *K_out = prefix;
    *kk_out = need;
}

// Writes the selected tokens of m keys (key_at, idx_at; idx ascending in i) in order:
// keys above K, and the first kk keys equal to K; pads the row to k with -1.
template <class KeyAt, class IdxAt>
__device__ void bs_write(KeyAt key_at, IdxAt idx_at, int m, int k, uint32_t K, int kk, int* wtot, int* orow) {
    int out_base = 0, eq_base = 0;
    for (int c0 = 0; c0 < m; c0 += kBsThreads) {
        const int i = c0 + threadIdx.x;
        const uint32_t key = i < m ? key_at(i) : 0u;
        const bool eq = i < m && key == K;
        int te;
        const int er = eq_base + bs_excl_scan(eq ? 1 : 0, wtot, &te);
        const bool s = i < m && (key > K || (eq && er < kk));
        int ts;
        const int pos = out_base + bs_excl_scan(s ? 1 : 0, wtot, &ts);
        if (s && pos < k) orow[pos] = idx_at(i);
        out_base += ts;
        eq_base += te;
    }
    for (int j = out_base + threadIdx.x; j < k; j += kBsThreads) orow[j] = -1;
}

__global__ void __launch_bounds__(kBsThreads)
    bin_final_kernel(const uint32_t* __restrict__ keys, long long ld, int n, int nblk, int k,
                     const uint32_t* __restrict__ ckey, const int* __restrict__ cidx, const int* __restrict__ ccnt,
                     int* __restrict__ out, WsHeader* hdr) {
    extern __shared__ __align__(16) unsigned char bs_smem[];
    uint32_t* skey = reinterpret_cast<uint32_t*>(bs_smem);
    int* sidx = reinterpret_cast<int*>(skey + kBsSmemCand);
    int* soff = sidx + kBsSmemCand;  // [nblk + 1] slice offsets
    __shared__ int sh[256];
    __shared__ int sel[2];
    __shared__ int wtot[kBsThreads / 32];
    const int row = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* orow = out + static_cast<long long>(row) * k;
    const uint32_t* kr = keys + row * ld;
    // slice offsets (slices are token ranges in order, so the kept keys stay in token order)
    int total = 0, over = 0;
    for (int c0 = 0; c0 < nblk; c0 += kBsThreads) {
        const int j = c0 + threadIdx.x;
        const int c = j < nblk ? ccnt[row * nblk + j] : 0;
        int t, o;
        const int off = total + bs_excl_scan(min(c, kBsSliceCap), wtot, &t);
        bs_excl_scan(c > kBsSliceCap ? 1 : 0, wtot, &o);
        if (j < nblk) soff[j] = off;
        total += t;
        over += o;
    }
    if (threadIdx.x == 0) soff[nblk] = total;
    const bool fast = over == 0 && total <= kBsSmemCand;
    __syncthreads();
    uint32_t K;
    int kk;
    if (fast) {
        // every kept key g in [0, total): its slice by binary search over the offsets, then the
        // load (independent loads, four in flight per thread)
        for (int g0 = 0; g0 < total; g0 += 4 * kBsThreads) {
            uint32_t kv[4];
            int iv[4], gv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int g = g0 + r * kBsThreads + static_cast<int>(threadIdx.x);
                gv[r] = g;
                kv[r] = 0u;
                iv[r] = 0;
                if (g < total) {
                    int lo = 0, hi = nblk - 1;  // the last slice j with soff[j] <= g
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (soff[mid] <= g) lo = mid; else hi = mid - 1;
                    }
                    const size_t src = static_cast<size_t>(row * nblk + lo) * kBsSliceCap + (g - soff[lo]);
                    kv[r] = __ldg(ckey + src);
                    iv[r] = __ldg(cidx + src);
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
                if (gv[r] < total) {
                    skey[gv[r]] = kv[r];
                    sidx[gv[r]] = iv[r];
                }
        }
        __syncthreads();
        auto key_at = [&](int i) { return skey[i]; };
        auto idx_at = [&](int i) { return sidx[i]; };
        bs_kth(key_at, total, k, sh, sel, &K, &kk);
        bs_write(key_at, idx_at, total, k, K, kk, wtot, orow);
        if (threadIdx.x == 0 && hdr) atomicMax(&hdr->sel_max_kept, total);
    } else {
        // the kept keys do not fit: select from the whole row
        auto key_at = [&](int i) { return __ldg(kr + i); };
        auto idx_at = [&](int i) { return i; };
        bs_kth(key_at, n, k, sh, sel, &K, &kk);
        bs_write(key_at, idx_at, n, k, K, kk, wtot, orow);
        if (threadIdx.x == 0 && hdr) atomicAdd(&hdr->sel_full_rows, 1);
    }
}

}  // namespace

// Slices per row: enough CTAs to cover the SMs about four times, slices of at least 4096 keys.
int radix_blocks(int rows, int n, int num_sms, int* per) {
    int nblk = (4 * num_sms + rows - 1) / rows;
    const int most = (n + 4095) / 4096;
    if (nblk > most) nblk = most;
    if (nblk < 1) nblk = 1;
    *per = (n + nblk - 1) / nblk;
    *per = (*per + kRxThreads - 1) / kRxThreads * kRxThreads;
    nblk = (n + *per - 1) / *per;
    return nblk < 1 ? 1 : nblk;
}

size_t radix_topk_scratch_bytes(int rows, int n, int num_sms) {
    int per = 0;
    const int nblk = radix_blocks(rows, n, num_sms, &per);
    return static_cast<size_t>(rows) * (sizeof(RadixRow) + kRxBins * sizeof(int)) +
           static_cast<size_t>(rows) * nblk * sizeof(int2);
}

// Bin select scratch: the histograms the producer fills (zeroed before it runs), then the
// slices' counts and their kept keys.
size_t bin_topk_hist_bytes(int rows) { return static_cast<size_t>(rows) * kBsBins * sizeof(int); }

size_t bin_topk_scratch_bytes(int rows, int n, int num_sms) {
    int per = 0;
    const size_t nb = static_cast<size_t>(rows) * radix_blocks(rows, n, num_sms, &per);
    return bin_topk_hist_bytes(rows) + nb * sizeof(int) + nb * kBsSliceCap * (sizeof(uint32_t) + sizeof(int));
}

// Top-k of `rows` rows of n keys (row stride ld) whose histograms of the top kBsBits bits are at
// the start of `scratch` -> out [rows, k] ascending tokens, then -1.
cudaError_t launch_bin_topk(const uint32_t* keys, long long ld, int rows, int n, int k, int* out, void* scratch,
                            WsHeader* hdr, int num_sms, cudaStream_t stream) {
    int per = 0;
    const int nblk = radix_blocks(rows, n, num_sms, &per);
    int* hist = static_cast<int*>(scratch);
    int* ccnt = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(scratch) + bin_topk_hist_bytes(rows));
    uint32_t* ckey = reinterpret_cast<uint32_t*>(ccnt + static_cast<size_t>(rows) * nblk);
    int* cidx = reinterpret_cast<int*>(ckey + static_cast<size_t>(rows) * nblk * kBsSliceCap);
    const size_t fsm = static_cast<size_t>(2 * kBsSmemCand + nblk + 1) * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(bin_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(fsm));
    if (e != cudaSuccess) return e;
    bin_compact_kernel<<<static_cast<unsigned>(rows) * nblk, kRxThreads, 0, stream>>>(keys, ld, n, nblk, per, k, hist,
                                                                                       ckey, cidx, ccnt);
    bin_final_kernel<<<rows, kBsThreads, fsm, stream>>>(keys, ld, n, nblk, k, ckey, cidx, ccnt, out, hdr);
    return cudaGetLastError();
}

// Top-k of `rows` rows of n keys (row stride ld) -> out [rows, k] ascending tokens, then -1.
cudaError_t launch_radix_topk(const uint32_t* keys, long long ld, int rows, int n, int k, int* out, void* scratch,
                              int num_sms, cudaStream_t stream) {
    int per = 0;
    const int nblk = radix_blocks(rows, n, num_sms, &per);
    RadixRow* rs = static_cast<RadixRow*>(scratch);
    int* hist = reinterpret_cast<int*>(rs + rows);
    int2* counts = reinterpret_cast<int2*>(hist + static_cast<size_t>(rows) * kRxBins);
    const unsigned grid = static_cast<unsigned>(rows) * nblk;
    radix_init_kernel<<<(rows * kRxBins + kRxThreads - 1) / kRxThreads, kRxThreads, 0, stream>>>(rs, hist, rows, k);
    for (int pass = 0; pass < kRxPasses; ++pass)
        radix_hist_kernel<<<grid, kRxThreads, 0, stream>>>(keys, ld, n, nblk, per, pass, k, rs, hist);
    radix_count_kernel<<<grid, kRxThreads, 0, stream>>>(keys, ld, n, nblk, per, k, rs, counts);
    radix_write_kernel<<<grid, kRxThreads, 0, stream>>>(keys, ld, n, nblk, per, k, rs, counts, out);
    return cudaGetLastError();
}

}  // namespace dsa
