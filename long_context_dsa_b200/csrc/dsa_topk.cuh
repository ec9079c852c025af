// dsa_topk.cuh -- streaming per-row top-k used by the fused indexer and by
// the standalone selection kernel.
//
// Selection rule (the top-k of the DSA indexer, [Term] "dot product +
// top-k"): the k largest scores of the row, ties to the lower token index,
// -0.0 equal to +0.0; output ascending by token index, then -1.
//
// A row's state is a candidate buffer of (key, index) pairs plus an
// admission threshold.  Scores arrive in any order; an arriving pair is
// kept iff it ranks above the current k-th candidate.  When the buffer
// nears its capacity the group of NT threads that owns the row prunes it
// to exactly k entries with a two-key radix select (8-bit digits on the
// score key, then on the index for ties at the boundary) and raises the
// threshold to the new k-th entry.  At the end the survivors are sorted
// by index and written.
//
// The buffer may live in shared or global memory (generic pointers).
#pragma once

#include "dsa_common.cuh"

namespace dsa {

static constexpr int kCandCap = 4096;  // candidates per row buffer

struct TopkRowState {  // shared memory, one per row in flight
    int count;
    uint32_t thr_key;  // admit (key, idx) iff key > thr_key || (key == thr_key && idx < thr_idx)
    int thr_idx;
    int pad;
};

struct TopkScratch {  // shared memory, one per selection group
    int hist[256];
    int warp_val[16];
    int sel_digit, sel_above, sel_equal, misc;
};

__device__ __forceinline__ void topk_row_init(TopkRowState* st) {
    st->count = 0;
    st->thr_key = 0u;
    st->thr_idx = 0x7fffffff;
}

__device__ __forceinline__ bool topk_admit(const TopkRowState* st, uint32_t key, int idx) {
    const uint32_t tk = st->thr_key;
    return key > tk || (key == tk && idx < st->thr_idx);
}

// Warp-aggregated append into a buffer of `cap` entries.  Every lane of
// the warp must call it.  Callers prune before a buffer can fill; an append
// past `cap` is dropped and flagged instead of written.
__device__ __forceinline__ void topk_append_warp(TopkRowState* st, uint32_t* ckey, int* cidx, uint32_t key,
                                                 int idx, bool admit, int cap, WsHeader* hdr) {
    const unsigned m = __ballot_sync(0xffffffffu, admit);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(&st->count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (admit) {
        const int pos = base + __popc(m & ((1u << lane) - 1u));
        if (pos < cap) {
            ckey[pos] = key;
            cidx[pos] = idx;
        } else {
            raise_status(hdr, DSA_STATUS_OVERFLOW, pos);
        }
    }
}

template <int NT>
struct TopkGroup {
    static_assert(NT % 32 == 0 && NT <= 512, "group of whole warps");
    static constexpr int PER = kCandCap / NT;
    static_assert(PER <= 32, "per-thread item mask is 32 bits");

    int tid;   // thread index within the group
    int bar;   // named barrier id reserved for the group
    TopkScratch* sc;
    int cap;   // entries in each row buffer (<= kCandCap)

    __device__ __forceinline__ void sync() const { named_bar_sync(bar, NT); }

    // kk-th largest (1-based) of the participating items v[i] (bit i of
    // `part`) over the whole group.  Returns it; n_greater / n_equal count
    // the participating items above / equal to it.
    __device__ uint32_t kth_largest(const uint32_t (&v)[PER], uint32_t part, int kk, int& n_greater,
                                    int& n_equal) const {
        uint32_t prefix = 0u, fixed = 0u;
        int above = 0, equal = 0;
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int b = tid; b < 256; b += NT) sc->hist[b] = 0;
            sync();
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                if (((part >> i) & 1u) && (v[i] & fixed) == prefix)
                    atomicAdd(&sc->hist[(v[i] >> shift) & 255u], 1);
            }
            sync();
            if (tid < 32) {
                const int lane = tid;
                int s8 = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) s8 += sc->hist[lane * 8 + j];
                int suf = s8;  // count in bins >= lane*8
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_down_sync(0xffffffffu, suf, off);
                    if (lane + off < 32) suf += o;
                }
                const unsigned ball = __ballot_sync(0xffffffffu, suf >= kk);
                const int L = 31 - __clz(ball);
                if (lane == L) {
                    int acc = suf - s8;
                    for (int j = 7; j >= 0; --j) {
                        const int c = sc->hist[L * 8 + j];
                        if (acc + c >= kk) {
                            sc->sel_digit = L * 8 + j;
                            sc->sel_above = acc;
                            sc->sel_equal = c;
                            break;
                        }
                        acc += c;
                    }
                }
            }
            sync();
            const int dsel = sc->sel_digit;
            kk -= sc->sel_above;
            above += sc->sel_above;
            equal = sc->sel_equal;
            prefix |= static_cast<uint32_t>(dsel) << shift;
            fixed |= 0xFFu << shift;
        }
        n_greater = above;
        n_equal = equal;
        return prefix;
    }

    // Exclusive prefix sum of `c` over the group; *total gets the sum.
    __device__ int excl_scan(int c, int* total) const {
        const int lane = tid & 31, w = tid >> 5;
        int inc = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) sc->warp_val[w] = inc;
        sync();
        int before = 0, tot = 0;
#pragma unroll
        for (int j = 0; j < NT / 32; ++j) {
            const int x = sc->warp_val[j];
            before += (j < w) ? x : 0;
            tot += x;
        }
        sync();
        *total = tot;
        return before + inc - c;
    }

    __device__ int max_reduce(int x) const {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, off));
        if ((tid & 31) == 0) sc->warp_val[tid >> 5] = x;
        sync();
        int r = sc->warp_val[0];
#pragma unroll
        for (int j = 1; j < NT / 32; ++j) r = max(r, sc->warp_val[j]);
        sync();
        return r;
    }

    // Keep exactly the k best candidates of the row (requires count > k).
    // All NT threads call it; st->count is read after a group barrier.
    __device__ void prune(TopkRowState* st, uint32_t* ckey, int* cidx, int k) const {
        const int n = min(st->count, cap);
        if (n <= k) return;  // nothing to drop (every thread reads the same n)
        uint32_t rk[PER];
        int ri[PER];
        uint32_t valid = 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int j = tid + i * NT;
            const bool ok = j < n;
            rk[i] = ok ? ckey[j] : 0u;
            ri[i] = ok ? cidx[j] : 0;
            valid |= (ok ? 1u : 0u) << i;
        }
        int G, E;
        const uint32_t kstar = kth_largest(rk, valid, k, G, E);  // includes barriers: loads are done
        const int kk = k - G;  // entries needed from key == kstar
        uint32_t eq = 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) eq |= ((((valid >> i) & 1u) && rk[i] == kstar) ? 1u : 0u) << i;
        uint32_t ithr = 0xffffffffu;  // keep key == kstar entries with idx <= ithr
        if (E > kk) {
            uint32_t nv[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) nv[i] = ~static_cast<uint32_t>(ri[i]);
            int g2, e2;
            ithr = ~kth_largest(nv, eq, kk, g2, e2);
        }
        uint32_t keep = 0u;
        int maxeq = -1;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const bool gt = ((valid >> i) & 1u) && rk[i] > kstar;
            const bool ke = ((eq >> i) & 1u) && static_cast<uint32_t>(ri[i]) <= ithr;
            keep |= ((gt || ke) ? 1u : 0u) << i;
            if (ke) maxeq = max(maxeq, ri[i]);
        }
        int total;
        int pos = excl_scan(__popc(keep), &total);  // barrier inside: every load above is done
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if ((keep >> i) & 1u) {
                ckey[pos] = rk[i];
                cidx[pos] = ri[i];
                ++pos;
            }
        }
        const int thr_idx = max_reduce(maxeq);
        if (tid == 0) {
            st->count = total;  // == k
            st->thr_key = kstar;
            st->thr_idx = thr_idx;
        }
        sync();
    }

    // Final selection of the row: prune to k if needed, sort the indices
    // ascending in `sortbuf` (shared, >= next_pow2(k) ints) and write
    // out[0..k) (then -1 padding).  All NT threads call it.
    __device__ void finish(TopkRowState* st, uint32_t* ckey, int* cidx, int k, int* out, int* sortbuf) const {
        sync();
        if (st->count > k) prune(st, ckey, cidx, k);
        const int n = min(st->count, k);
        int P = 1;
        while (P < n) P <<= 1;
        for (int j = tid; j < P; j += NT) sortbuf[j] = (j < n) ? cidx[j] : 0x7fffffff;
        sync();
        for (int size = 2; size <= P; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int i = tid; i < (P >> 1); i += NT) {
                    const int lo = (i / stride) * stride * 2 + (i % stride);
                    const int hi = lo + stride;
                    const int a = sortbuf[lo], b = sortbuf[hi];
                    const bool asc = (lo & size) == 0;
                    if ((a > b) == asc) {
                        sortbuf[lo] = b;
                        sortbuf[hi] = a;
                    }
                }
                sync();
            }
        }
        for (int j = tid; j < k; j += NT) out[j] = (j < n) ? sortbuf[j] : -1;
        sync();
    }
};

}  // namespace dsa
