// dsa_topk_radix.cu -- per-row top-k of a few long rows of score keys (one-query decode).
//
// Same selection rule as every other top-k in the library ([Term] "dot product + top-k"; ties
// to the lower token index, output ascending then -1).  For a decode step over a contiguous
// cache the one-query indexer writes its row of order-preserving score keys (4 bytes per cached
// token: 51 MB for 64 rows of 200K tokens, 4 MB for one row of 1M) and, while it scores, counts
// the keys' top bits into a histogram per row.  The selection then needs one pass over the keys:
//   * compaction: each slice CTA finds the histogram bin that holds its row's k-th key and keeps
//     its keys from that bin up, in token order (fewer than k above the bin, plus the bin);
//   * final: one CTA per row selects among the kept keys in shared memory (the exact k-th key is
//     searched among the keys of its bin alone, equal keys taken in token order) and writes the
//     tokens in order.
// A row whose kept keys do not fit (scores packed into one bin, many equal scores) is selected by
// the same CTA from its whole row.  No CTA ever waits for another: the steps are separate launches.
#include "dsa_common.cuh"

namespace dsa {

namespace {

constexpr int kRxThreads = 256;
// Block-wide exclusive scan of two counts over kRxThreads threads (every thread gets its offsets).
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

// ---------------------------------------------------------------------------------------------
// Bin select: the same result for rows whose producer also counted their keys into a histogram of
// the top kBsBits bits (sign, 8 exponent bits, 4 mantissa bits of the score).
//   * compaction: every slice CTA finds the bin T holding its row's k-th largest key from the
//     histogram (suffix counts), then keeps its keys whose bin is >= T, in token order, in its own
//     region (at most kBsSliceCap) -- fewer than k keys above T plus the keys of bin T.
//   * final: one CTA per row loads the row's kept keys (at most kBsSmemCand) into shared memory in
//     token order.  The compaction recorded T and the number of keys above it, so the k-th key K
//     is the (k - above)-th largest key of bin T: a radix select over those keys' low
//     32 - kBsBits bits finds it and how many keys equal to K to take.  The CTA then writes the
//     selected tokens in order.  A row whose kept keys overflow
//     either bound (a score distribution packed into a few bins, many equal scores) is selected
//     by the same CTA directly from the full row instead.
constexpr int kBsBits = kBinTopkBits;
constexpr int kBsBins = 1 << kBsBits;
constexpr int kBsShift = 32 - kBsBits;
constexpr int kBsThreads = 512;
constexpr int kBsSliceCap = 2048;
constexpr int kBsSmemCand = 16384;

// The largest bin T with count(bins >= T) >= k in one row's histogram, and the count of keys in
// the bins above it (T = 0, above = -1 when the row holds fewer than k keys: everything is kept);
// every thread of the kRxThreads-thread block gets them.
__device__ int bs_threshold_bin(const int* __restrict__ h, int k, int* hs, int* tsum, int* res, int* above_out) {
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
    if (t == 0) {
        res[0] = 0;
        res[1] = -1;
    }
    __syncthreads();
    int later = 0;  // keys in the warps above this one
    for (int j = w + 1; j < kRxThreads / 32; ++j) later += tsum[j];
    suf += later;
    const int above_me = suf - s;
    if (suf >= k && above_me < k) {
        int acc = above_me, T = t * PB;
        for (int j = PB - 1; j >= 0; --j) {
            const int c = hs[t * PB + j];
            if (acc + c >= k) {
                T = t * PB + j;
                break;
            }
            acc += c;
        }
        res[0] = T;
        res[1] = acc;  // keys in bins above T
    }
    __syncthreads();
    const int T = res[0];
    *above_out = res[1];
    __syncthreads();
    return T;
}

// Keys in row `row`: n, or its own length clamped to [1, cap] when the rows differ.
__device__ __forceinline__ int bs_row_len(int n, const int* lens, int cap, int row) {
    if (!lens) return n;
    const int len = __ldg(lens + row);
    return len < 1 ? 1 : (len > cap ? cap : len);
}

// Keys of one slice with bin >= T, in token order, into the slice's region; the slice's count
// (uncapped: a count above kBsSliceCap marks the row for the whole-row select).  Each thread
// takes 8 consecutive keys of a 2048-key chunk, a block scan orders the kept keys, and a running
// base carries across chunks.
__global__ void __launch_bounds__(kRxThreads)
    bin_compact_kernel(const uint32_t* __restrict__ keys, long long ld, int n, const int* __restrict__ lens,
                       int len_cap, int nblk, int per, int k, const int* __restrict__ hist,
                       uint32_t* __restrict__ ckey, int* __restrict__ cidx, int* __restrict__ ccnt,
                       int2* __restrict__ rinfo) {
    __shared__ int2 wt[kRxThreads / 32];
    __shared__ int tsum[kRxThreads / 32];
    __shared__ int res[2];
    __shared__ __align__(16) int hs[kBsBins];
    const int row = blockIdx.x / nblk, blk = blockIdx.x % nblk;
    const uint32_t* kr = keys + row * ld;
    const int nr = bs_row_len(n, lens, len_cap, row);
    const int i0 = blk * per, i1 = min(nr, i0 + per);
    // 8 consecutive keys of the chunk at c0 for this thread (two 16-byte loads when aligned)
    auto load8 = [&](int c0, uint32_t (&kv)[8]) {
        const int a = c0 + threadIdx.x * 8;
        if (a + 8 <= i1 && ((row * ld + a) & 3) == 0) {
            const uint4 x = __ldg(reinterpret_cast<const uint4*>(kr + a));
            const uint4 y = __ldg(reinterpret_cast<const uint4*>(kr + a + 4));
            kv[0] = x.x; kv[1] = x.y; kv[2] = x.z; kv[3] = x.w;
            kv[4] = y.x; kv[5] = y.y; kv[6] = y.z; kv[7] = y.w;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) kv[e] = a + e < i1 ? __ldg(kr + a + e) : 0u;
        }
    };
    uint32_t nx[8];
    load8(i0, nx);  // the first chunk's keys load while the threshold is found
    int above;
    const uint32_t T = static_cast<uint32_t>(
        bs_threshold_bin(hist + static_cast<size_t>(row) * kBsBins, k, hs, tsum, res, &above));
    if (blk == 0 && threadIdx.x == 0) rinfo[row] = make_int2(static_cast<int>(T), above);
    uint32_t* ok = ckey + static_cast<size_t>(blockIdx.x) * kBsSliceCap;
    int* oi = cidx + static_cast<size_t>(blockIdx.x) * kBsSliceCap;
    int base = 0;
    for (int c0 = i0; c0 < i1; c0 += kRxThreads * 8) {
        const int a = c0 + threadIdx.x * 8;
        uint32_t kv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[e] = nx[e];
        if (c0 + kRxThreads * 8 < i1) load8(c0 + kRxThreads * 8, nx);  // the next chunk loads during this one
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

// The need-th largest of the keys produced by key_at(i) (i < m) whose bits from lo_bit up equal
// `prefix`, and how many of the keys equal to it are selected; passes of up to 8 bits from bit
// lo_bit - 1 down, each with a shared-memory histogram.  (lo_bit = 32, prefix = 0: all m keys.)
template <class KeyAt>
__device__ void bs_kth(KeyAt key_at, int m, int need, uint32_t prefix, int lo_bit, int* sh, int* sel,
                       uint32_t* K_out, int* kk_out) {
    while (lo_bit > 0) {
        const int width = lo_bit < 8 ? lo_bit : 8;
        const int shift = lo_bit - width;
        const uint32_t fixed = lo_bit >= 32 ? 0u : (0xffffffffu << lo_bit);
        const uint32_t dmask = (1u << width) - 1u;
        lo_bit = shift;
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
                const uint32_t dg = (key >> shift) & dmask;
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
    bin_final_kernel(const uint32_t* __restrict__ keys, long long ld, int n, const int* __restrict__ lens,
                     int len_cap, int nblk, int k, const uint32_t* __restrict__ ckey, const int* __restrict__ cidx,
                     const int* __restrict__ ccnt, const int2* __restrict__ rinfo, int* __restrict__ out,
                     WsHeader* hdr) {
    extern __shared__ __align__(16) unsigned char bs_smem[];
    uint32_t* skey = reinterpret_cast<uint32_t*>(bs_smem);
    int* sidx = reinterpret_cast<int*>(skey + kBsSmemCand);
    int* soff = sidx + kBsSmemCand;  // [nblk + 1] slice offsets
    __shared__ int sh[256];
    __shared__ int sel[2];
    __shared__ int wtot[kBsThreads / 32];
    const int row = blockIdx.x;
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
        // the k-th key lies in bin T, below `above` keys of the higher bins: only bin T's keys and
        // their low bits are left to search (every key is kept when the row holds fewer than k)
        const int2 ri = rinfo[row];
        if (ri.y < 0)
            bs_kth(key_at, total, min(k, total), 0u, 32, sh, sel, &K, &kk);
        else
            bs_kth(key_at, total, k - ri.y, static_cast<uint32_t>(ri.x) << kBsShift, kBsShift, sh, sel, &K, &kk);
        bs_write(key_at, idx_at, total, k, K, kk, wtot, orow);
        if (threadIdx.x == 0 && hdr) atomicMax(&hdr->sel_max_kept, total);
    } else {
        // the kept keys do not fit: select from the whole row
        const int nr = bs_row_len(n, lens, len_cap, row);
        auto key_at = [&](int i) { return __ldg(kr + i); };
        auto idx_at = [&](int i) { return i; };
        bs_kth(key_at, nr, min(k, nr), 0u, 32, sh, sel, &K, &kk);
        bs_write(key_at, idx_at, nr, k, K, kk, wtot, orow);
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

// Bin select scratch: the histograms the producer fills (zeroed before it runs), then the
// slices' counts and their kept keys.
size_t bin_topk_hist_bytes(int rows) { return static_cast<size_t>(rows) * kBsBins * sizeof(int); }

size_t bin_topk_scratch_bytes(int rows, int n, int num_sms) {
    int per = 0;
    const size_t nb = static_cast<size_t>(rows) * radix_blocks(rows, n, num_sms, &per);
    return bin_topk_hist_bytes(rows) + nb * sizeof(int) + nb * kBsSliceCap * (sizeof(uint32_t) + sizeof(int)) +
           static_cast<size_t>(rows) * sizeof(int2);
}

// Top-k of `rows` rows of n keys (row stride ld; with `lens`, row r holds its own length clamped
// to [1, len_cap]) whose histograms of the top kBsBits bits are at the start of `scratch`
// -> out [rows, k] ascending tokens, then -1.
cudaError_t launch_bin_topk(const uint32_t* keys, long long ld, int rows, int n, int k, int* out, void* scratch,
                            WsHeader* hdr, const int* lens, int len_cap, int num_sms, cudaStream_t stream) {
    int per = 0;
    const int nblk = radix_blocks(rows, n, num_sms, &per);
    // hist | rinfo (8-byte records: right after the histograms, whose size is a multiple of 8) |
    // ccnt | ckey | cidx
    int* hist = static_cast<int*>(scratch);
    int2* rinfo = reinterpret_cast<int2*>(reinterpret_cast<unsigned char*>(scratch) + bin_topk_hist_bytes(rows));
    int* ccnt = reinterpret_cast<int*>(rinfo + rows);
    uint32_t* ckey = reinterpret_cast<uint32_t*>(ccnt + static_cast<size_t>(rows) * nblk);
    int* cidx = reinterpret_cast<int*>(ckey + static_cast<size_t>(rows) * nblk * kBsSliceCap);
    const size_t fsm = static_cast<size_t>(2 * kBsSmemCand + nblk + 1) * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(bin_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(fsm));
    if (e != cudaSuccess) return e;
    bin_compact_kernel<<<static_cast<unsigned>(rows) * nblk, kRxThreads, 0, stream>>>(
        keys, ld, n, lens, len_cap, nblk, per, k, hist, ckey, cidx, ccnt, rinfo);
    bin_final_kernel<<<rows, kBsThreads, fsm, stream>>>(keys, ld, n, lens, len_cap, nblk, k, ckey, cidx, ccnt, rinfo,
                                                        out, hdr);
    return cudaGetLastError();
}

}  // namespace dsa
