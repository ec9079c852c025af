// dsa_topk.cuh -- streaming per-row top-k used by the fused indexer and by
// the standalone selection kernel.
//
// Selection rule (the top-k of the DSA indexer, [Term] "dot product +
// top-k"): the k largest scores of the row, ties to the lower token index,
// -0.0 equal to +0.0; output ascending by token index, then -1.
//
// A row is owned by a group of NT threads (NW = NT/32 warps).  Its
// candidate buffer of `cap` (key, index) pairs is split into NW
// sub-buffers, one per warp, so a warp appends with a ballot and a count
// it keeps in a register -- no atomics.  Callers feed each warp its keys in
// ascending token order, so every sub-buffer stays sorted by index.  An
// arriving pair is appended iff it ranks above the row's admission
// threshold (the current k-th candidate).  When a sub-buffer nears its
// share the group prunes the row to exactly k entries: a radix select over
// the order-preserving score key that starts at the highest bit where the
// candidates differ (8-bit digits, per-warp histograms), then over the
// index for ties at the boundary.  Each warp compacts its own survivors in
// place, in order (coalesced, and the sub-buffers stay sorted); only if one
// warp would keep too many to leave room for further appends are the
// survivors merged into index order and split evenly over the sub-buffers
// (still sorted: later appends carry larger indices).  The threshold rises
// to the new k-th entry.  At the end the row is written by merging its
// sub-buffers: each entry's output position is its rank in its own list
// plus its binary-searched ranks in the others.
//
// Buffers may live in shared or global memory (generic pointers).
#pragma once

#include "dsa_common.cuh"

namespace dsa {

static constexpr int kCandCap = 4096;  // largest candidate buffer per row

struct TopkRowState {  // shared memory, one per row in flight
    uint32_t thr_key;  // admit (key, idx) iff key > thr_key || (key == thr_key && idx < thr_idx)
    int thr_idx;
    int cnt[4];        // per-warp sub-buffer counts, published at check points
};

template <int NW>
struct TopkScratchT {  // shared memory, one per selection group
    int hist[NW][256];
    int warp_val[NW];
    int sel_digit, sel_above, sel_equal, misc;
};

__device__ __forceinline__ void topk_row_init(TopkRowState* st) {
    st->thr_key = 0u;
    st->thr_idx = 0x7fffffff;
    st->cnt[0] = st->cnt[1] = st->cnt[2] = st->cnt[3] = 0;
}

// Warp append into this warp's sub-buffer (`sub` entries at ckey/cidx).
// Every lane of the warp must call it; `cnt` is the warp's (uniform) count.
// Entries past the sub-buffer are dropped (callers prune before that can
// happen); `cnt` still counts them, so the caller can report an overflow.
__device__ __forceinline__ void topk_append_warp(uint32_t* ckey, int* cidx, int& cnt, uint32_t key, int idx,
                                                 bool admit, int sub) {
    const unsigned m = __ballot_sync(0xffffffffu, admit);
    const int pos = cnt + __popc(m & ((1u << (threadIdx.x & 31)) - 1u));
    const uint32_t doit = static_cast<uint32_t>(admit & (pos < sub));
    // predicated stores: no divergent branch around them
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.u32 p, %0, 0;\n\t"
        "@p st.u32 [%1], %3;\n\t"
        "@p st.u32 [%2], %4;\n\t}" ::"r"(doit),
        "l"(ckey + pos), "l"(cidx + pos), "r"(key), "r"(idx)
        : "memory");
    cnt += __popc(m);
}

template <int NT>
struct TopkGroup {
    static constexpr int NW = NT / 32;
    static constexpr int PER = kCandCap / NT;  // items per thread when a row is loaded
    static_assert(NT % 32 == 0 && NW <= 4, "group of at most 4 warps");
    static_assert(PER <= 32, "per-thread item mask is 32 bits");
    using Scratch = TopkScratchT<NW>;

    int tid;   // thread index within the group
    int bar;   // named barrier id reserved for the group
    Scratch* sc;
    int cap;   // entries in each row buffer (<= kCandCap, a multiple of NT)

    __device__ __forceinline__ void sync() const { named_bar_sync(bar, NT); }
    __device__ __forceinline__ int sub() const { return cap / NW; }
    __device__ __forceinline__ int warp() const { return tid >> 5; }

    __device__ int sum_reduce(int x) const {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if ((tid & 31) == 0) sc->warp_val[tid >> 5] = x;
        sync();
        int r = 0;
#pragma unroll
        for (int j = 0; j < NW; ++j) r += sc->warp_val[j];
        sync();
        return r;
    }
    __device__ uint32_t umax_reduce(uint32_t x) const {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, off));
        if ((tid & 31) == 0) sc->warp_val[tid >> 5] = static_cast<int>(x);
        sync();
        uint32_t r = 0u;
#pragma unroll
        for (int j = 0; j < NW; ++j) r = max(r, static_cast<uint32_t>(sc->warp_val[j]));
        sync();
        return r;
    }

    // Over the summed per-warp histograms of 256 bins: the bin holding the
    // kk-th largest item (sel_digit), the count above it (sel_above) and in it
    // (sel_equal).  Threads 0-31 work; the caller syncs before and after.
    __device__ void scan_bins(int kk) const {
        if (tid < 32) {
            const int lane = tid;
            int cnt8[8];
            int s8 = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                int c = 0;
#pragma unroll
                for (int ww = 0; ww < NW; ++ww) c += sc->hist[ww][lane * 8 + j];
                cnt8[j] = c;
                s8 += c;
            }
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
    }

    // kk-th largest (1-based, kk <= number of participants) of the
    // participating items v[i] (bit i of `part`) over the whole group.
    // n_greater / n_equal count the participants above / equal to it.
    __device__ uint32_t kth_largest(const uint32_t (&v)[PER], uint32_t part, int kk, int& n_greater,
                                    int& n_equal) const {
        // the digits start at the highest bit where participants differ
        uint32_t hi = 0u, lo_inv = 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if ((part >> i) & 1u) {
                hi = max(hi, v[i]);
                lo_inv = max(lo_inv, ~v[i]);
            }
        }
        hi = umax_reduce(hi);
        const uint32_t lo = ~umax_reduce(lo_inv);
        const uint32_t diff = hi ^ lo;
        if (diff == 0u) {  // every participant is equal
            n_greater = 0;
            n_equal = sum_reduce(__popc(part));
            return hi;
        }
        int nbits = 32 - __clz(diff);  // bits below the common prefix
        uint32_t fixed = nbits >= 32 ? 0u : ~((1u << nbits) - 1u);
        uint32_t prefix = hi & fixed;
        int above = 0, equal = 0;
        const int w = warp();
#pragma unroll 1
        while (nbits > 0) {
            const int width = nbits < 8 ? nbits : 8;
            const int shift = nbits - width;
            const uint32_t dmask = (1u << width) - 1u;
            for (int b = tid; b < NW * 256; b += NT) (&sc->hist[0][0])[b] = 0;
            sync();
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                if (((part >> i) & 1u) && (v[i] & fixed) == prefix) atomicAdd(&sc->hist[w][(v[i] >> shift) & dmask], 1);
            }
            sync();
            scan_bins(kk);
            sync();
            const int dsel = sc->sel_digit;
            kk -= sc->sel_above;
            above += sc->sel_above;
            equal = sc->sel_equal;
            prefix |= static_cast<uint32_t>(dsel) << shift;
            fixed |= dmask << shift;
            nbits = shift;
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
        for (int j = 0; j < NW; ++j) {
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
        for (int j = 1; j < NW; ++j) r = max(r, sc->warp_val[j]);
        sync();
        return r;
    }

    // This thread's share of the row: entries lane, lane+32, ... of its warp's sub-buffer.
    __device__ void load_own(const TopkRowState* st, const uint32_t* ckey, const int* cidx, uint32_t (&rk)[PER],
                             int (&ri)[PER], uint32_t& valid) const {
        const int w = warp(), lane = tid & 31, s = sub();
        const int n = min(st->cnt[w], s);
        const uint32_t* kk = ckey + w * s;
        const int* ii = cidx + w * s;
        valid = 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int j = lane + 32 * i;
            const bool ok = j < n;
            rk[i] = ok ? kk[j] : 0u;
            ri[i] = ok ? ii[j] : 0;
            valid |= (ok ? 1u : 0u) << i;
        }
    }

    // Keep exactly the k best candidates of the row and raise the threshold.
    // A warp keeps its survivors in its own sub-buffer, in order, when every
    // warp keeps at most `keep_max`; otherwise they are dealt round-robin.
    // All NT threads call it after a group barrier that follows the
    // publication of st->cnt.
    __device__ void prune(TopkRowState* st, uint32_t* ckey, int* cidx, int k, int keep_max, int* sortbuf) const {
        int total0 = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) total0 += min(st->cnt[w], sub());
        if (total0 <= k) return;  // nothing to drop (every thread reads the same counts)
        uint32_t rk[PER];
        int ri[PER];
        uint32_t valid;
        load_own(st, ckey, cidx, rk, ri, valid);
        int G, E;
        const uint32_t kstar = kth_largest(rk, valid, k, G, E);  // barriers inside: all loads are done
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
        const int w = warp(), lane = tid & 31, s = sub();
        const unsigned lt = (1u << lane) - 1u;
        // this warp's survivors, counted in sub-buffer order
        int wkeep = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) wkeep += __popc(__ballot_sync(0xffffffffu, (keep >> i) & 1u));
        if (lane == 0) sc->warp_val[w] = wkeep;
        sync();  // every load above is done before any store below
        int wmax = 0, total = 0;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) {
            wmax = max(wmax, sc->warp_val[ww]);
            total += sc->warp_val[ww];
        }
        sync();
        if (wmax <= keep_max) {
            // compact in place, in order: coalesced and still sorted by index
            int b = 0;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const unsigned m = __ballot_sync(0xffffffffu, (keep >> i) & 1u);
                if ((keep >> i) & 1u) {
                    const int pos = b + __popc(m & lt);
                    ckey[w * s + pos] = rk[i];
                    cidx[w * s + pos] = ri[i];
                }
                b += __popc(m);
            }
        } else {
            // one warp holds too many survivors to keep appending: merge all survivors into
            // index order and split them evenly over the sub-buffers
            int off[NW + 1];
            off[0] = 0;
            for (int ww = 0; ww < NW; ++ww) off[ww + 1] = off[ww] + sc_counts(ww);
            int b = 0;
#pragma unroll
            for (int i = 0; i < PER; ++i) {  // this warp's survivor indices, in order, into sortbuf
                const unsigned m = __ballot_sync(0xffffffffu, (keep >> i) & 1u);
                if (((keep >> i) & 1u) && off[w] + b + __popc(m & lt) < k) sortbuf[off[w] + b + __popc(m & lt)] = ri[i];
                b += __popc(m);
            }
            sync();
            total = min(total, k);
            const int qn = (total + NW - 1) / NW;  // survivors per sub-buffer after the split
            b = 0;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const unsigned m = __ballot_sync(0xffffffffu, (keep >> i) & 1u);
                if ((keep >> i) & 1u) {
                    int r = b + __popc(m & lt);
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww)
                        if (ww != w) r += lower_rank(sortbuf + off[ww], min(off[ww + 1], k) - min(off[ww], k), ri[i]);
                    if (r < total) {
                        const int dw = r / qn, slot = r - dw * qn;
                        ckey[dw * s + slot] = rk[i];
                        cidx[dw * s + slot] = ri[i];
                    }
                }
                b += __popc(m);
            }
        }
        const int thr_idx = max_reduce(maxeq);
        if (tid == 0) {
            st->thr_key = kstar;
            st->thr_idx = thr_idx;
        }
        if (wmax <= keep_max) {
            if (lane == 0) st->cnt[w] = wkeep;
        } else if (tid == 0) {
            const int qn = (total + NW - 1) / NW;
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) st->cnt[ww] = max(0, min(qn, total - ww * qn));
        }
        sync();
    }

    // Streaming prune: keeps, in place and in order, every candidate whose key
    // is at least a threshold T chosen so that at least k and at most
    // k + slack candidates qualify -- a superset of the row's current top k,
    // so nothing that can still be selected is dropped -- and raises the
    // admission threshold to T (ties at T are admitted).  T is the lower edge
    // of the bin that holds the k-th key in a 256-bin histogram over the key
    // range [current threshold, largest key], refined inside that bin until
    // it is small enough; usually one pass against the several digit passes
    // of an exact select.  Falls back to the exact prune when one key value
    // carries more ties than the slack, or when one warp would keep more than
    // keep_max.  Same calling rules as prune.
    __device__ void prune_fast(TopkRowState* st, uint32_t* ckey, int* cidx, int k, int keep_max, int slack,
                               int* sortbuf) const {
        int total0 = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) total0 += min(st->cnt[w], sub());
        if (total0 <= k) return;
        uint32_t rk[PER];
        int ri[PER];
        uint32_t valid;
        load_own(st, ckey, cidx, rk, ri, valid);
        uint32_t lo = st->thr_key;  // every candidate's key is at least the threshold it passed
        uint32_t hi = 0u, lo_inv = 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if ((valid >> i) & 1u) {
                hi = max(hi, rk[i]);
                lo_inv = max(lo_inv, ~rk[i]);
            }
        }
        hi = umax_reduce(hi);
        if (lo == 0u) lo = ~umax_reduce(lo_inv);  // first prune of the row (uniform: lo is shared)
        const int w = warp(), lane = tid & 31, s_ = sub();
        int above = 0, kk = k;
        uint32_t T = lo;
        bool exact = false;
#pragma unroll 1
        while (true) {
            const uint32_t span = hi - lo;
            const int sh = span < 256u ? 0 : (32 - __clz(span)) - 8;  // bins of 2^sh keys
            for (int b = tid; b < NW * 256; b += NT) (&sc->hist[0][0])[b] = 0;
            sync();
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                if (((valid >> i) & 1u) && rk[i] >= lo && rk[i] <= hi) atomicAdd(&sc->hist[w][(rk[i] - lo) >> sh], 1);
            }
            sync();
            scan_bins(kk);
            sync();
            const uint32_t blo = lo + (static_cast<uint32_t>(sc->sel_digit) << sh);
            const int ab = sc->sel_above, eqc = sc->sel_equal;
            above += ab;
            kk -= ab;
            if (above + eqc <= k + slack) {  // keep the whole bin
                T = blo;
                break;
            }
            if (sh == 0) {  // one key value with more ties than the slack
                exact = true;
                break;
            }
            const uint32_t wmask = (1u << sh) - 1u;
            hi = (hi - blo > wmask) ? blo + wmask : hi;
            lo = blo;
        }
        if (exact) {
            prune(st, ckey, cidx, k, keep_max, sortbuf);
            return;
        }
        uint32_t keep = 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) keep |= ((((valid >> i) & 1u) && rk[i] >= T) ? 1u : 0u) << i;
        const unsigned lt = (1u << lane) - 1u;
        int wkeep = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) wkeep += __popc(__ballot_sync(0xffffffffu, (keep >> i) & 1u));
        if (lane == 0) sc->warp_val[w] = wkeep;
        sync();  // every load above is done before any store below
        int wmax = 0;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) wmax = max(wmax, sc->warp_val[ww]);
        sync();
        if (wmax > keep_max) {
            prune(st, ckey, cidx, k, keep_max, sortbuf);
            return;
        }
        int b = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const unsigned m = __ballot_sync(0xffffffffu, (keep >> i) & 1u);
            if ((keep >> i) & 1u) {
                const int pos = b + __popc(m & lt);
                ckey[w * s_ + pos] = rk[i];
                cidx[w * s_ + pos] = ri[i];
            }
            b += __popc(m);
        }
        if (tid == 0) {
            st->thr_key = T;
            st->thr_idx = 0x7fffffff;
        }
        if (lane == 0) st->cnt[w] = wkeep;
        sync();
    }

    // Survivor count of warp ww, as published in the scratch during prune.
    __device__ __forceinline__ int sc_counts(int ww) const { return sc->warp_val[ww]; }

    // Number of entries of the ascending list a[0..n) that are < x.
    __device__ static __forceinline__ int lower_rank(const int* a, int n, int x) {
        int lo = 0, hi = n;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (a[mid] < x)
                lo = mid + 1;
            else
                hi = mid;
        }
        return lo;
    }

    // Final selection of the row: prune to k if needed, then write the
    // survivors ascending by index to out_idx[0..k) (then -1 padding) and,
    // if out_key is not NULL, their score keys to out_key (then 0).  Uses
    // `sortbuf` (shared, >= k ints).  All NT threads call it after a group
    // barrier that follows the publication of st->cnt.
    __device__ void finish(TopkRowState* st, uint32_t* ckey, int* cidx, int k, int* out_idx, uint32_t* out_key,
                           int* sortbuf) const {
        prune(st, ckey, cidx, k, sub(), sortbuf);
        const int w = warp(), lane = tid & 31, s = sub();
        // concatenate the NW ascending lists in sortbuf, then place every entry at its rank
        // in its own list plus its ranks in the other lists
        int off[NW + 1];
        off[0] = 0;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) off[ww + 1] = off[ww] + min(min(st->cnt[ww], s), k - off[ww]);
        const int n = off[NW];
        for (int j = lane; j < off[w + 1] - off[w]; j += 32) sortbuf[off[w] + j] = cidx[w * s + j];
        sync();
        for (int e = tid; e < n; e += NT) {
            int le = 0;
#pragma unroll
            for (int ww = 1; ww < NW; ++ww) le += (e >= off[ww]) ? 1 : 0;
            const int x = sortbuf[e];
            int pos = e - off[le];
#pragma unroll
            for (int ww = 0; ww < NW; ++ww)
                if (ww != le) pos += lower_rank(sortbuf + off[ww], off[ww + 1] - off[ww], x);
            if (pos < k) {
                out_idx[pos] = x;
                if (out_key) out_key[pos] = ckey[le * s + (e - off[le])];
            }
        }
        for (int j = n + tid; j < k; j += NT) {
            out_idx[j] = -1;
            if (out_key) out_key[j] = 0u;
        }
        sync();
    }
};

}  // namespace dsa
