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
