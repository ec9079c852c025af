// dsa_latent_tc.cu -- sparse attention over shared latent rows (MLA-style) on the sm_100a
// tensor cores: the prefill form, for many query rows with 64 query heads each.
//
// Operation ([Explainer] §稀疏注意力的隐性开销: each token attends only to its top-k history
// tokens; the latent layout is this library's reading for the 1M-token configuration): one
// 576-dim bf16 row per token is the key of every query head, its first 512 dims the value.
//     O[t,h] = sum_{j in I[t]} softmax_j(scale * Q[t,h] . R[j]) R[j][:512]
//
// B200 design.  One unit = one query row's 64 heads; its top-k list is cut into tiles of 64
// selected tokens.
//   * Gather: TMA tile::gather4 (no multicast) pulls 4 selected 1152-byte rows at a time,
//     in nine 128-byte column blocks, straight into the 128-byte swizzled K-major layout the
//     tensor core reads; 2 stages of 72 KB.
//   * S = Q R^T: tcgen05.mma kind::f16, M = 64 heads, N = 64 tokens, K = 576 (36 K-steps),
//     A = the query block (resident, 72 KB), B = the gathered tile; fp32 S in TMEM (two
//     buffers of 64 columns, so S of the next tile runs while the softmax reads this one).
//   * Softmax: one thread per head reads its S row from TMEM, keeps a running max that is
//     raised only when it grows by more than 2^8 (the accumulated O is then rescaled in TMEM;
//     rare), and writes P as bf16 hi + lo parts (about 16 significant bits) to shared memory.
//   * O^T += V^T P^T: M = 512 value dims (4 MMAs of M = 128), N = 64 heads, K = 64 tokens;
//     A = the same gathered tile read MN-major (the value dims of a token are contiguous),
//     B = P^T (K-major); P_hi lands in the tile's rope block (dims 512-575, free once S is
//     done), P_lo in its own buffer.  O^T stays in TMEM (256 columns) for the whole row.
//   * Warp roles: warps 0-3 softmax and epilogue (TMEM lane quadrants 0-3), warp 4 TMA
//     producer, warp 5 MMA issuer.  Persistent CTAs walk the units.
//   * Every wait is bounded; on a timeout the kernel flags DSA_STATUS_TIMEOUT and winds down.
#include <cuda.h>

#include "dsa_tc.cuh"

namespace dsa {
cudaError_t launch_latent_merge(const float* part, int HB, int hblocks, int splits, long long units, int Hq, void* O,
                                bool out_bf16, cudaStream_t stream);
namespace lattc {

constexpr int DQK = 576, DV = 512, HB = 64, NK = 64;
constexpr int NBLK = DQK / 64;              // 9 column blocks of 64 dims (128 bytes)
constexpr int BLK = NK * 128;               // one column block of a tile (64 rows x 128 B)
constexpr int TILE = NBLK * BLK;            // 73728 bytes
constexpr int OFF_Q = 0;
constexpr int OFF_ST = OFF_Q + NBLK * HB * 128;   // 2 stages
constexpr int OFF_PLO = OFF_ST + 2 * TILE;
constexpr int OFF_ALPHA = OFF_PLO + HB * NK * 2;  // float[64]
constexpr int OFF_L = OFF_ALPHA + HB * 4;         // float[64]
constexpr int OFF_BAR = OFF_L + HB * 4;
constexpr int NBAR = 16;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;        // + alignment slack
static_assert(SMEM <= 232448, "shared memory budget");

constexpr int SCOL = 0;     // S buffers: columns 0 and 64
constexpr int OCOL = 128;   // O^T tiles: columns 128 + 64 t, t = 0..3
constexpr float kRescaleLog2 = 8.0f;

// 128-byte swizzled shared-memory descriptor with explicit strides.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Four rows (r0..r3) x 64 columns starting at column x of a 2-D tensor map with a one-row box.
__device__ __forceinline__ void tma_gather4(void* smem_dst, const CUtensorMap* map, int x, int r0, int r1, int r2,
                                            int r3, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
    uint32_t(&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
    tc::tmem_ld32(taddr, a);
    tc::tmem_ld32(taddr + 32, b);
    tc::tmem_wait_ld_dep(a);
    tc::tmem_wait_ld_dep(b);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16 TMEM lanes (of this warp's quadrant) x 32 columns, twice: threads 0-15 read lanes 0-15 at
// columns [col, col+32), threads 16-31 the same lanes at [col+32, col+64).  An M = 64 accumulator
// keeps its rows in lanes 0-15 of each quadrant, so the whole warp shares one S row block.
__device__ __forceinline__ void tmem_ld_16x32bx2(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Non-blocking: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// OR of `pred` over the `n` threads that meet at named barrier `id`.
__device__ __forceinline__ bool bar_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of row r, 16-byte chunk c in a 128-byte swizzled block of 128-byte rows.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

struct Params {
    const int* idx;
    int B, n_q, n_kv, Hq, topk, hblocks;
    int splits, tps;  // each unit's tiles in `splits` ranges of `tps` tiles (1 range: no split)
    float* part;      // splits > 1: per (item, head) unnormalised O^T, max and sum; merged afterwards
    float scale_log2;
    void* O;
    IdxShare share;
    WsHeader* hdr;
};

template <bool OUT_BF16>
__global__ void __launch_bounds__(192, 1)
    latent_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kv,
                     const Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sQ = smem + OFF_Q;
    unsigned char* sSt = smem + OFF_ST;
    unsigned char* sPlo = smem + OFF_PLO;
    float* sAlpha = reinterpret_cast<float*>(smem + OFF_ALPHA);
    float* sL = reinterpret_cast<float*>(smem + OFF_L);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* kv_full = bars + 2;   // [2]
    uint64_t* kv_empty = bars + 4;  // [2]
    uint64_t* s_full = bars + 6;    // [2]
    uint64_t* s_empty = bars + 8;   // [2]
    uint64_t* p_full = bars + 10;
    uint64_t* o_done = bars + 11;
    uint64_t* o_free = bars + 12;
    uint64_t* drain = bars + 13;
    uint64_t* plo_free = bars + 14;  // the P_lo half of a PV is done: P_lo may be rewritten
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long units = static_cast<long long>(p.B) * p.n_q * p.hblocks;
    const long long items = units * p.splits;
    const int ntiles = (p.topk + NK - 1) / NK;
    // item -> (unit, first tile, tiles): a unit's tiles are cut into ranges when units are few
    auto item_tiles = [&](long long it, long long& u, int& t0, int& nt) {
        u = it / p.splits;
        t0 = static_cast<int>(it % p.splits) * p.tps;
        nt = min(ntiles, t0 + p.tps) - t0;
    };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], 128);
        }
        mbar_init(p_full, 128);
        mbar_init(o_done, 1);
        mbar_init(plo_free, 1);
        mbar_init(o_free, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        tc::prefetch_tmap(&tmap_q);
        tc::prefetch_tmap(&tmap_kv);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&](int site) {
        raise_status(p.hdr, DSA_STATUS_TIMEOUT, site);
        *abort_flag = 1;
    };

    // token of entry kk of unit u's index row, -1 when skipped (padding, beyond the query's own
    // position for shared rows, or out of range -- the last flagged by the producer)
    auto entry = [&](const int* irow, int lim, int kk) -> int {
        if (kk >= p.topk) return -1;
        const int t = __ldg(irow + kk);
        return (t >= 0 && t < p.n_kv && t <= lim) ? t : -1;
    };
    auto unit_row = [&](long long u, long long& row, int& hb, const int*& irow, int& lim, long long& b) {
        row = u / p.hblocks;
        hb = static_cast<int>(u % p.hblocks);
        b = row / p.n_q;
        const int qi = static_cast<int>(row - b * p.n_q);
        irow = p.idx + (b * p.share.rows(p.n_q) + qi / p.share.q_per_idx) * static_cast<long long>(p.topk);
        lim = p.share.limit(qi);
    };

    if (warp == 4) {
        // ======================================================== TMA producer (whole warp)
        uint32_t g = 0, uc = 0;
        int q_issued = -1;  // last unit whose query block was requested (lane 0)
        bool ok = true;
        for (long long it = blockIdx.x; it < items && ok; it += gridDim.x, ++uc) {
            long long u, row, b;
            int hb, lim, t0, nt;
            const int* irow;
            item_tiles(it, u, t0, nt);
            unit_row(u, row, hb, irow, lim, b);
            if (lane == 0) {
                if (uc > 0 && !mbar_wait(q_empty, (uc - 1) & 1)) { fail(0x4c01); ok = false; }
                if (ok && *abort_flag) ok = false;
                if (ok) {
                    mbar_arrive_expect_tx(q_full, NBLK * HB * 128);
                    const int y = static_cast<int>(row * p.Hq + hb * HB);
                    for (int c = 0; c < NBLK; ++c) tc::tma_load_2d(sQ + c * HB * 128, &tmap_q, c * 64, y, q_full);
                    q_issued = uc;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            for (int j = 0; j < nt && ok; ++j, ++g) {
                const int st = g & 1;
                // lane: 4 keys (group kg) and half of the 9 column blocks; the index reads go out
                // before the wait for the stage, so their latency hides behind it
                const int kg = lane & 15;
                int r[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kk = (t0 + j) * NK + kg * 4 + i;
                    r[i] = kk < p.topk ? __ldg(irow + kk) : -1;
                }
                if (lane == 0) {
                    if (g >= 2 && !mbar_wait(&kv_empty[st], ((g >> 1) - 1) & 1)) { fail(0x4c02); ok = false; }
                    if (ok && *abort_flag) ok = false;
                    if (ok) mbar_arrive_expect_tx(&kv_full[st], TILE);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = r[i];
                    if ((t < -1 || t >= p.n_kv) && lane < 16) raise_status(p.hdr, DSA_STATUS_BAD_INDEX, t);
                    const bool v = t >= 0 && t < p.n_kv && t <= lim;
                    r[i] = static_cast<int>(b * p.n_kv + (v ? t : 0));  // skipped entries read row 0 (masked)
                }
                unsigned char* stg = sSt + st * TILE;
                const int c0 = lane < 16 ? 0 : 5, c1 = lane < 16 ? 5 : NBLK;
                for (int c = c0; c < c1; ++c)
                    tma_gather4(stg + c * BLK + kg * 4 * 128, &tmap_kv, c * 64, r[0], r[1], r[2], r[3], &kv_full[st]);
            }
        }
        // never leave with TMA writes in flight into shared memory
        if (lane == 0) {
            // the last query block and the last two tiles requested (already landed in a normal run)
            if (q_issued >= 0) mbar_wait(q_full, static_cast<uint32_t>(q_issued) & 1);
            for (uint32_t k2 = (g > 2 ? g - 2 : 0); k2 < g; ++k2) mbar_wait(&kv_full[k2 & 1], (k2 >> 1) & 1);
        }
    } else if (warp == 5) {
        // ======================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::make_idesc(1, 1, 64, 64);
            constexpr uint32_t idesc_o = tc::make_idesc(1, 1, 128, 64) | (1u << 15);  // A (V^T) MN-major
            uint32_t g = 0, pc = 0, uc = 0;
            bool ok = true;
            // S(j+1) and PV(j) wait on different things (the gather of tile j+1, the softmax of tile
            // j); the issuer polls both and issues whichever is ready, so a slow gather never holds
            // back a PV that could free a stage for the next gather.
            for (long long it = blockIdx.x; it < items && ok; it += gridDim.x, ++uc) {
                long long u;
                int t0, nt;
                item_tiles(it, u, t0, nt);
                if (!mbar_wait(q_full, uc & 1)) { fail(0x4c11); break; }
                const uint32_t g0 = g;
                int ns = 0, np = 0;  // next S and next PV of this item
                uint64_t idle0 = 0;
                while (np < nt) {
                    bool prog = false;
                    if (ns < nt && ns <= np + 1) {
                        const uint32_t gt = g0 + ns;
                        const int st = gt & 1, bb = gt & 1;
                        if (mbar_test(&kv_full[st], (gt >> 1) & 1) &&
                            (gt < 2 || mbar_test(&s_empty[bb], ((gt >> 1) - 1) & 1))) {
                            tc::fence_after_sync();
                            const uint32_t a0 = smem_u32(sQ), b0 = smem_u32(sSt + st * TILE);
#pragma unroll 1
                            for (int c = 0; c < NBLK; ++c)
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    tc::mma_f16(tmem + SCOL + bb * 64, sdesc(a0 + c * HB * 128 + kk * 32, 16, 1024),
                                                sdesc(b0 + c * BLK + kk * 32, 16, 1024), idesc_s, (c | kk) != 0);
                            tc::mma_commit(&s_full[bb]);
                            ++ns;
                            if (ns == nt) tc::mma_commit(q_empty);  // every S of the item issued
                            prog = true;
                        }
                    }
                    if (np < ns && mbar_test(p_full, pc & 1) &&
                        (np > 0 || uc == 0 || mbar_test(o_free, (uc - 1) & 1))) {
                        ++pc;
                        tc::fence_after_sync();
                        const int st = (g0 + np) & 1;
                        const uint32_t v0 = smem_u32(sSt + st * TILE);
                        const uint32_t phi = v0 + (NBLK - 1) * BLK, plo = smem_u32(sPlo);
                        // the P_lo products first, so the softmax may refill P_lo while the P_hi
                        // products still run
#pragma unroll 1
                        for (int t = 0; t < 4; ++t)
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                tc::mma_f16(tmem + OCOL + t * 64, sdesc(v0 + 2 * t * BLK + ks * 2048, BLK, 1024),
                                            sdesc(plo + ks * 32, 16, 1024), idesc_o, (np | ks) != 0);
                        tc::mma_commit(plo_free);
#pragma unroll 1
                        for (int t = 0; t < 4; ++t)
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                tc::mma_f16(tmem + OCOL + t * 64, sdesc(v0 + 2 * t * BLK + ks * 2048, BLK, 1024),
                                            sdesc(phi + ks * 32, 16, 1024), idesc_o, true);
                        tc::mma_commit(&kv_empty[st]);
                        tc::mma_commit(o_done);
                        ++np;
                        prog = true;
                    }
                    if (prog) {
                        idle0 = 0;
                    } else {
                        __nanosleep(32);  // leave the issue slots to the softmax warp sharing this sub-partition
                        const uint64_t now = globaltimer_ns();
                        if (idle0 == 0) {
                            idle0 = now;
                        } else if (now - idle0 > kWaitLimitNs || *abort_flag) {
                            if (!*abort_flag) fail(0x4c14);
                            ok = false;
                            break;
                        }
                    }
                }
                g += nt;
            }
            // nothing may still run on the tensor core when TMEM is released
            tc::mma_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ======================================================== softmax + epilogue (warps 0-3)
        // Each head's S row (64 tokens) is shared by two lanes: lanes 0-15 take tokens 0-31 of heads
        // 16q..16q+15, lanes 16-31 tokens 32-63 of the same heads (tcgen05.ld 16x32bx2).
        const int q = warp;                    // TMEM lane quadrant
        const int hl = lane & 15, half = lane >> 4;
        const int h = 16 * q + hl;             // this thread's head
        const bool lead = half == 0;           // writes the head's per-head values
        const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t sb = 0, oc = 0, uc = 0;
        bool ok = true, pv_waited = false;
        for (long long it = blockIdx.x; it < items && ok; it += gridDim.x, ++uc) {
            long long u, row, b;
            int hb, lim, t0, nt;
            const int* irow;
            item_tiles(it, u, t0, nt);
            unit_row(u, row, hb, irow, lim, b);
            float m_run = -INFINITY, l_run = 0.f;
            // entries of the current tile (lane i: entry i and 32 + i), read one tile ahead
            int e0 = entry(irow, lim, t0 * NK + lane), e1 = entry(irow, lim, t0 * NK + 32 + lane);
            for (int j = 0; j < nt; ++j, ++sb) {
                const uint32_t live0 = __ballot_sync(0xffffffffu, e0 >= 0);
                const uint32_t live1 = __ballot_sync(0xffffffffu, e1 >= 0);
                if (j + 1 < nt) {
                    e0 = entry(irow, lim, (t0 + j + 1) * NK + lane);
                    e1 = entry(irow, lim, (t0 + j + 1) * NK + 32 + lane);
                }
                const uint32_t live = half ? live1 : live0;  // this lane's 32 tokens
                const int bb = sb & 1;
                const bool got = mbar_wait(&s_full[bb], (sb >> 1) & 1);
                if (bar_or(1, 128, !got)) {
                    if (lane == 0 && !got) fail(0x4c21);
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                uint32_t v[32];
                tmem_ld_16x32bx2(tq + SCOL + bb * 64, v);
                tc::tmem_wait_ld_dep(v);
                tc::fence_before_sync();
                mbar_arrive(&s_empty[bb]);
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float sv = ((live >> i) & 1u) ? __uint_as_float(v[i]) * p.scale_log2 : -INFINITY;
                    v[i] = __float_as_uint(sv);
                    mx = fmaxf(mx, sv);
                }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run, mx);
                bool resc = false;
                float alpha = 1.f;
                if (j == 0 || m_run == -INFINITY) {
                    m_run = m_new;  // nothing accumulated yet for this head (O column is zero)
                } else if (m_new > m_run + kRescaleLog2) {
                    resc = true;
                    alpha = exp2f(m_run - m_new);
                    m_run = m_new;
                    l_run *= alpha;
                }
                const bool any = bar_or(2, 128, resc);
                // P = 2^(s - m_run), as bf16 hi + lo; a row of P^T (64 tokens of head h) is 128 bytes,
                // this lane's half is its 16-byte chunks 4 half .. 4 half + 3
                uint32_t hi[16], lo[16];
                float lsum = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float s0 = __uint_as_float(v[2 * i]), s1 = __uint_as_float(v[2 * i + 1]);
                    const float p0 = (m_run == -INFINITY) ? 0.f : exp2f(s0 - m_run);
                    const float p1 = (m_run == -INFINITY) ? 0.f : exp2f(s1 - m_run);
                    lsum += p0 + p1;
                    hi[i] = pack_bf16x2(p0, p1);
                    const __nv_bfloat162 hh = *reinterpret_cast<const __nv_bfloat162*>(&hi[i]);
                    lo[i] = pack_bf16x2(p0 - __low2float(hh), p1 - __high2float(hh));
                }
                l_run += lsum + __shfl_xor_sync(0xffffffffu, lsum, 16);
                // P_hi goes to the rope block of this tile's stage: every role walks the same units and
                // tiles, so the producer's and the MMA issuer's tile counter equals sb here
                unsigned char* phi = sSt + (sb & 1) * TILE + (NBLK - 1) * BLK;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(phi + sw128(h, 4 * half + c)) =
                        make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                if (j > 0) {
                    // the previous tile's PV has read P_lo (its P_lo products come first); with a
                    // rescale the whole PV must be done, so that O^T is stable
                    bool got2 = mbar_wait(plo_free, (oc - 1) & 1);
                    if (got2 && any) {
                        got2 = mbar_wait(o_done, (oc - 1) & 1);
                        pv_waited = true;
                    }
                    if (bar_or(1, 128, !got2)) {
                        if (lane == 0 && !got2) fail(0x4c22);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    if (any) {
                        if (lead) sAlpha[h] = resc ? alpha : 1.f;
                        named_bar_sync(3, 128);
                        for (int t = 0; t < 4; ++t) {
                            uint32_t o[64];
                            tmem_ld64(tq + OCOL + t * 64, o);
#pragma unroll
                            for (int i = 0; i < 64; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * sAlpha[i]);
                            tmem_st32(tq + OCOL + t * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                            tmem_st32(tq + OCOL + t * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                        }
                        tmem_wait_st();
                        named_bar_sync(3, 128);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(sPlo + sw128(h, 4 * half + c)) =
                        make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                fence_proxy_async_smem();  // P (generic writes) before the tensor core reads it
                tc::fence_before_sync();
                mbar_arrive(p_full);
                if (j > 0 && !pv_waited) {
                    // consume the previous PV's completion in order (its products are done by now)
                    const bool got3 = mbar_wait(o_done, (oc - 1) & 1);
                    if (bar_or(1, 128, !got3)) {
                        if (lane == 0 && !got3) fail(0x4c24);
                        ok = false;
                        break;
                    }
                }
                pv_waited = false;
                ++oc;  // oc: PVs issued so far, this tile's included
            }
            if (!ok) break;
            // ---- epilogue: O = O^T / l, written row-major [head][d]
            const bool got = mbar_wait(o_done, (oc - 1) & 1);
            if (bar_or(1, 128, !got)) {
                if (lane == 0 && !got) fail(0x4c23);
                break;
            }
            tc::fence_after_sync();
            if (p.part) {
                // a range of the unit's tiles: unnormalised O^T and (max, sum) per head, [item][head][DV + 2]
                float* pb = p.part + static_cast<size_t>(it) * HB * (DV + 2);
                if (lead) {
                    pb[static_cast<size_t>(h) * (DV + 2) + DV] = m_run;
                    pb[static_cast<size_t>(h) * (DV + 2) + DV + 1] = l_run;
                }
                for (int t = 0; t < 4; ++t) {
                    uint32_t o[64];
                    tmem_ld64(tq + OCOL + t * 64, o);
                    const int d = t * 128 + q * 32 + lane;
#pragma unroll
                    for (int i = 0; i < 64; ++i) pb[static_cast<size_t>(i) * (DV + 2) + d] = __uint_as_float(o[i]);
                }
                tc::fence_before_sync();
                named_bar_sync(3, 128);
                mbar_arrive(o_free);
                continue;
            }
            if (lead) sL[h] = l_run > 0.f ? 1.f / l_run : 0.f;
            named_bar_sync(3, 128);
            const size_t obase = (static_cast<size_t>(row) * p.Hq + static_cast<size_t>(hb) * HB) * DV;
            for (int t = 0; t < 4; ++t) {
                uint32_t o[64];
                tmem_ld64(tq + OCOL + t * 64, o);
                const int d = t * 128 + q * 32 + lane;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float val = __uint_as_float(o[i]) * sL[i];
                    if (OUT_BF16)
                        reinterpret_cast<__nv_bfloat16*>(p.O)[obase + static_cast<size_t>(i) * DV + d] =
                            __float2bfloat16_rn(val);
                    else
                        reinterpret_cast<float*>(p.O)[obase + static_cast<size_t>(i) * DV + d] = val;
                }
            }
            tc::fence_before_sync();
            named_bar_sync(3, 128);  // every thread has read sL before the next unit rewrites it
            mbar_arrive(o_free);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [rows, 576] bf16 rows, 128-byte swizzled boxes of 64 columns x box_rows.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &qr) !=
                cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(DQK), rows};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(DQK) * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lattc

// The tensor-core form serves query heads in blocks of 64.  With fewer (row, head block) units
// than SMs (decode) each unit's tiles are cut into ranges, at most `max_splits` (the warp-MMA
// kernel's split count for the same shape, which sizes the workspace), merged afterwards.
bool latent_tc_applies(int Hq) { return Hq % lattc::HB == 0; }

cudaError_t launch_latent_tc(const void* Q, const void* KV, const int* idx, int B, int n_q, int n_kv, int Hq,
                             int topk, float scale, void* O, bool out_bf16, IdxShare share, WsHeader* hdr,
                             int max_splits, int num_sms, cudaStream_t stream) {
    using namespace lattc;
    CUtensorMap mq, mkv;
    if (!make_map(&mq, Q, static_cast<uint64_t>(B) * n_q * Hq, HB) ||
        !make_map(&mkv, KV, static_cast<uint64_t>(B) * n_kv, 1))
        return cudaErrorInvalidValue;
    Params p;
    p.idx = idx;
    p.B = B;
    p.n_q = n_q;
    p.n_kv = n_kv;
    p.Hq = Hq;
    p.topk = topk;
    p.hblocks = Hq / HB;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.O = O;
    p.share = share;
    p.hdr = hdr;
    const long long units = static_cast<long long>(B) * n_q * p.hblocks;
    const int ntiles = (topk + NK - 1) / NK;
    int splits = 1;
    if (units < num_sms && max_splits > 1) {
        splits = static_cast<int>((num_sms + units - 1) / units);
        if (splits > max_splits) splits = max_splits;
        if (splits > ntiles) splits = ntiles;
    }
    p.tps = (ntiles + splits - 1) / splits;
    p.splits = (ntiles + p.tps - 1) / p.tps;
    p.part = p.splits > 1 ? reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(hdr) + kWsHeaderBytes) : nullptr;
    auto kern = out_bf16 ? latent_tc_kernel<true> : latent_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    const long long items = units * p.splits;
    const int grid = items < num_sms ? static_cast<int>(items) : num_sms;
    kern<<<grid, 192, SMEM, stream>>>(mq, mkv, p);
    if ((e = cudaGetLastError()) != cudaSuccess || p.splits == 1) return e;
    return launch_latent_merge(p.part, HB, p.hblocks, p.splits, units, Hq, O, out_bf16, stream);
}

}  // namespace dsa
