// dsa_indexer.cu -- fused indexer scores + streaming top-k (K1 + K2) on
// the sm_100a tensor cores.
//
// Operation: the DSA lightning indexer ([QbitAI] §IndexCache: a light
// indexer before each attention layer scans the context and picks the
// important tokens; [Term]: "dot product + top-k"):
//     score[t,s] = sum_h w[t,h] * ReLU(q_I[t,h,:] . k_I[s,:]),  s <= t,
// then the top-k of each row (ties to the lower index), written as
// ascending indices.  The L x L score matrix never leaves the SM.
//
// B200 design
//   * GEMM shape: keys on M (128 per tile, TMEM lanes), (query, head)
//     pairs on N (256 per accumulator), d_I on K.  Each epilogue thread
//     owns one key (one TMEM lane) and reduces over heads in registers:
//     no cross-thread reduction.
//   * One work tile = 2 groups of 256/H_I queries sharing every key tile:
//     two 128x256 fp32 accumulators fill all 512 TMEM columns and
//     ping-pong between the MMA and the two epilogue warpgroups, and each
//     128-key tile fetched by TMA feeds 2 MMAs (halving L2 traffic).
//   * Warp roles: warps 0-3 epilogue group 0, 4-7 epilogue group 1,
//     warp 8 TMA producer, warp 9 MMA issuer (+ TMEM allocation).
//   * Operands are staged by TMA (no multicast) with 128-byte swizzle; the
//     query tile stays resident while the key tiles stream.
//   * Epilogue: tcgen05.ld -> ReLU -> x w -> sum over heads -> causal
//     mask -> admission test against the row's running top-k threshold ->
//     warp-aggregated append to the row's candidate buffer (global scratch,
//     L2-resident) -> prune when the buffer nears capacity: one histogram pass
//     keeps a superset of the k best (an exact radix select when ties crowd
//     one bin), and an exact prune to k ends each row.
//   * Persistent CTAs take work tiles longest-first in a snake order so the
//     causal triangle balances across SMs.
//   * Every wait is bounded (DSA_STATUS_TIMEOUT instead of a hang).
#include <cuda.h>

#include "dsa_tc.cuh"
#include "dsa_topk.cuh"

namespace dsa {

template <int H, int D, bool FP8>
struct IdxCfg {
    static constexpr int ESZ = FP8 ? 1 : 2;
    static constexpr int ROWB = D * ESZ;        // bytes per operand row
    static constexpr int KB = ROWB / 128;       // 128-byte swizzle blocks per row
    static constexpr int KSTEPS = ROWB / 32;    // MMA K-steps (32 bytes of K each)
    static constexpr int QG = 256 / H;          // queries per accumulator group
    static constexpr int QT = 2 * QG;           // queries per work tile
    static constexpr int A_STAGE = 128 * ROWB;  // one key tile
    static constexpr int B_GROUP = 256 * ROWB;  // one query group tile
    static constexpr int STAGES = (ROWB == 256) ? 2 : 4;
    static constexpr int BOX_X = 128 / ESZ;     // elements per 128-byte TMA box row
    static constexpr int THREADS = 320;
    static constexpr int OFF_B = 0;
    static constexpr int OFF_A = OFF_B + 2 * B_GROUP;
    static constexpr int OFF_W = OFF_A + STAGES * A_STAGE;
    static constexpr int OFF_ST = OFF_W + 2 * 256 * 4;
    static constexpr int OFF_SC = OFF_ST + 2 * QG * static_cast<int>(sizeof(TopkRowState));
    static constexpr int OFF_SORT = OFF_SC + 2 * static_cast<int>(sizeof(TopkGroup<128>::Scratch));
    static constexpr int OFF_BAR = OFF_SORT + 2 * DSA_TOPK_MAX * 4;
    static constexpr int NBAR = 2 + 2 * STAGES + 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_NEED = OFF_MISC + 16;  // [2 parities][2 groups][need, soft] prune masks
    static constexpr int SMEM = OFF_NEED + 64 + 1024;  // + alignment slack
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(D * ESZ % 128 == 0, "rows must be whole 128-byte swizzle blocks");
};

struct IdxParams {
    const float* w;
    const float* q_scale;
    const float* k_scale;
    int B, n_q, q_pos0, n_kv, topk, cap;
    int tiles_per_b, n_tiles;
    int* idx_out;
    uint32_t* cand;  // [grid][2][QG][2*cap]
    float* scores;   // score-output mode: [B, n_q, n_kv]
    WsHeader* hdr;
};

// Work tile for round r of CTA c: longest tiles first, snake over CTAs.
__device__ __forceinline__ int tile_index(int c, int r, int G) { return r * G + ((r & 1) ? (G - 1 - c) : c); }

// SCORES = false: fused top-k (the product path).  SCORES = true: write the
// causal scores instead of selecting (test/debug export; same MMA and
// epilogue arithmetic).
template <int H, int D, bool FP8, bool SCORES>
__global__ void __launch_bounds__(320, 1)
    indexer_topk_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const IdxParams p) {
    using C = IdxCfg<H, D, FP8>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled operand tiles, by offsetting the shared array itself
    // (an integer round trip would make every later access a generic one)
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sB = smem + C::OFF_B;
    unsigned char* sA = smem + C::OFF_A;
    float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
    TopkRowState* sSt = reinterpret_cast<TopkRowState*>(smem + C::OFF_ST);
    auto* sSc = reinterpret_cast<TopkGroup<128>::Scratch*>(smem + C::OFF_SC);
    int* sSort = reinterpret_cast<int*>(smem + C::OFF_SORT);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* kv_full = bars + 2;
    uint64_t* kv_empty = kv_full + C::STAGES;
    uint64_t* acc_full = kv_empty + C::STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
    int* wg_abort = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);  // [2], written only by each group
    unsigned long long* sNeed = reinterpret_cast<unsigned long long*>(smem + C::OFF_NEED);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(&acc_full[g], 1);
            mbar_init(&acc_empty[g], 128);
        }
        *abort_flag = 0;
        wg_abort[0] = wg_abort[1] = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        tc::prefetch_tmap(&tmap_q);
        tc::prefetch_tmap(&tmap_k);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 8) {
        // ================================================== TMA producer
        if (lane == 0) {
            uint32_t it = 0, wt = 0;
            bool ok = true;
            int pend_q = -1;
            const bool withhold = test_withhold_tile(p.hdr);  // timeout test: first key tile never sent
            for (int r = 0; ok; ++r) {
                const int ti = tile_index(blockIdx.x, r, G);
                if (ti >= p.n_tiles) break;
                const int qt = p.tiles_per_b - 1 - ti / p.B;
                const int b = ti % p.B;
                const int q0 = qt * C::QT;
                const int nvq = min(C::QT, p.n_q - q0);
                const int nkt = (p.q_pos0 + q0 + nvq + 127) / 128;
                if (wt > 0 && !mbar_wait(q_empty, (wt - 1) & 1)) { ok = false; break; }
                mbar_arrive_expect_tx(q_full, 2 * C::B_GROUP);
                for (int g = 0; g < 2; ++g)
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_2d(sB + g * C::B_GROUP + kb * 256 * 128, &tmap_q, kb * C::BOX_X,
                                        (b * p.n_q + q0 + g * C::QG) * H, q_full);
                pend_q = static_cast<int>(wt);
                for (int j = 0; j < nkt; ++j, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t rr = it / C::STAGES;
                    if (rr > 0 && !mbar_wait(&kv_empty[s], (rr - 1) & 1)) { ok = false; break; }
                    if (withhold && it == 0) continue;  // nothing issued: the waits on this stage run out
                    mbar_arrive_expect_tx(&kv_full[s], C::A_STAGE);
                    for (int kb = 0; kb < C::KB; ++kb)
                        tc::tma_load_2d(sA + s * C::A_STAGE + kb * 128 * 128, &tmap_k, kb * C::BOX_X,
                                        b * p.n_kv + j * 128, &kv_full[s]);
                    if (*reinterpret_cast<volatile int*>(abort_flag)) { ok = false; ++it; break; }
                }
                ++wt;
            }
            if (!ok) {
                raise_status(p.hdr, DSA_STATUS_TIMEOUT, 0x1d01);
                atomicExch(abort_flag, 1);
            }
            // drain: never leave with TMA writes in flight into shared memory
            if (pend_q >= 0) mbar_wait(q_full, pend_q & 1);
            for (uint32_t k2 = (it > C::STAGES ? it - C::STAGES : 0); k2 < it; ++k2)
                mbar_wait(&kv_full[k2 % C::STAGES], (k2 / C::STAGES) & 1);
        }
    } else if (warp == 9) {
        // ================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = FP8 ? tc::make_idesc(0, 0, 128, 256) : tc::make_idesc(1, 1, 128, 256);
            uint32_t it = 0, wt = 0, u = 0;
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int ti = tile_index(blockIdx.x, r, G);
                if (ti >= p.n_tiles) break;
                const int qt = p.tiles_per_b - 1 - ti / p.B;
                const int q0 = qt * C::QT;
                const int nvq = min(C::QT, p.n_q - q0);
                const int nkt = (p.q_pos0 + q0 + nvq + 127) / 128;
                if (!mbar_wait(q_full, wt & 1)) { ok = false; break; }
                tc::fence_after_sync();
                for (int j = 0; j < nkt; ++j, ++it, ++u) {
                    const int s = it % C::STAGES;
                    if (!mbar_wait(&kv_full[s], (it / C::STAGES) & 1)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t a0 = smem_u32(sA + s * C::A_STAGE);
                    for (int g = 0; g < 2; ++g) {
                        if (u > 0 && !mbar_wait(&acc_empty[g], (u - 1) & 1)) { ok = false; break; }
                        tc::fence_after_sync();
                        const uint32_t b0 = smem_u32(sB + g * C::B_GROUP);
#pragma unroll
                        for (int ks = 0; ks < C::KSTEPS; ++ks) {
                            const uint32_t aoff = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
                            const uint32_t boff = (ks >> 2) * (256 * 128) + (ks & 3) * 32;
                            const uint64_t ad = tc::make_sdesc_sw128(a0 + aoff);
                            const uint64_t bd = tc::make_sdesc_sw128(b0 + boff);
                            if (FP8)
                                tc::mma_f8(tmem_base + g * 256, ad, bd, idesc, ks > 0);
                            else
                                tc::mma_f16(tmem_base + g * 256, ad, bd, idesc, ks > 0);
                        }
                        tc::mma_commit(&acc_full[g]);
                    }
                    if (!ok) break;
                    tc::mma_commit(&kv_empty[s]);
                    if (*reinterpret_cast<volatile int*>(abort_flag)) { ok = false; break; }
                }
                tc::mma_commit(q_empty);
                ++wt;
            }
            if (!ok) {
                raise_status(p.hdr, DSA_STATUS_TIMEOUT, 0x1d02);
                atomicExch(abort_flag, 1);
            }
        }
    } else {
        // ================================================== epilogue groups
        const int g = warp >> 2;            // accumulator / query group
        const int tid = threadIdx.x & 127;  // thread within the group == key lane
        const int wq = warp & 3;            // TMEM lane quadrant
        TopkGroup<128> grp{tid, 1 + g, &sSc[g], p.cap};
        float* ws = sW + g * 256;
        TopkRowState* st = sSt + g * C::QG;
        int* sortbuf = sSort + g * DSA_TOPK_MAX;
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + g * 256;
        constexpr int CHECK = 8;                       // prune checks every CHECK key tiles
        const int sub = grp.sub();                     // this warp's share of a row buffer
        const int room = sub - CHECK * 32;             // prune once a sub-buffer holds more than this
        const int slack = max(32, p.topk / 8);         // a prune may keep up to k + slack candidates
        // a row past this fill is pruned early when the other group stalls the MMA for a prune anyway
        const int soft_room = (room + (p.topk + slack) / 4) / 2;
        uint32_t chk = 0;                              // check points passed (same count in both groups)
        uint32_t u = 0;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const int ti = tile_index(blockIdx.x, r, G);
            if (ti >= p.n_tiles) break;
            const int qt = p.tiles_per_b - 1 - ti / p.B;
            const int b = ti % p.B;
            const int q0 = qt * C::QT;
            const int nvq = min(C::QT, p.n_q - q0);
            const int nkt = (p.q_pos0 + q0 + nvq + 127) / 128;
            const int qg0 = q0 + g * C::QG;  // first query row of this group
            // head weights of this group's queries (fp8: folded with q_scale)
            for (int c = tid; c < 256; c += 128) {
                const int q = c / H, h = c % H;
                float wv = 0.f;
                if (qg0 + q < p.n_q) {
                    const size_t o = (static_cast<size_t>(b) * p.n_q + qg0 + q) * H + h;
                    wv = p.w[o];
                    if (FP8) wv *= p.q_scale[o];
                }
                ws[c] = wv;
            }
            if (tid < C::QG) topk_row_init(&st[tid]);
            grp.sync();
            uint32_t* cbase = p.cand + (static_cast<size_t>(blockIdx.x) * 2 + g) * C::QG * 2 * p.cap;
            uint32_t* wkey = cbase + wq * sub;                              // row 0, this warp's keys
            int* widx = reinterpret_cast<int*>(cbase + p.cap) + wq * sub;  // row 0, this warp's indices
            const int rstride = 2 * p.cap;                                  // 32-bit words per row
            int cnt[C::QG];  // this warp's sub-buffer counts (warp-uniform; published at checks)
#pragma unroll
            for (int q = 0; q < C::QG; ++q) cnt[q] = 0;
            // rows of this group that exist, and the last key each may see
            const int qlast = min(C::QG, p.n_q - qg0);
            const int pos0 = p.q_pos0 + qg0;

            for (int j = 0; j < nkt; ++j, ++u) {
                // fp8: this key's scale, read before the wait so its latency hides behind it
                const int s_key0 = j * 128 + tid;
                const float ksc = (FP8 && s_key0 < p.n_kv) ? __ldg(p.k_scale + static_cast<size_t>(b) * p.n_kv + s_key0)
                                                            : 0.f;
                const bool got = __all_sync(0xffffffffu, mbar_wait(&acc_full[g], u & 1));
                if (!got) {
                    if (lane == 0) {
                        raise_status(p.hdr, DSA_STATUS_TIMEOUT, 0x1d03);
                        atomicExch(abort_flag, 1);
                        wg_abort[g] = 1;
                    }
                } else {
                    tc::fence_after_sync();
                    // score[q] = sum_h w[q,h] * ReLU(acc[q,h]) with packed fp32x2 FMAs; each
                    // 32-column chunk holds whole queries' heads (H >= 32: part of one query;
                    // H < 32: 32/H queries), so it is folded into sc[] as soon as it is done
                    float sc[C::QG];
#pragma unroll
                    for (int q = 0; q < C::QG; ++q) sc[q] = 0.f;
                    uint32_t va[32], vb[32];
                    tc::tmem_ld32(tbase, va);
                    tc::tmem_wait_ld_dep(va);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t(&cur)[32] = (c & 1) ? vb : va;
                        uint32_t(&nxt)[32] = (c & 1) ? va : vb;
                        if (c + 1 < 8) tc::tmem_ld32(tbase + (c + 1) * 32, nxt);
                        constexpr int NA = H >= 32 ? 4 : 32 / H;  // accumulators per chunk
                        unsigned long long a2[NA];
#pragma unroll
                        for (int e = 0; e < NA; ++e) a2[e] = 0ull;
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const ulonglong2 w4 = *reinterpret_cast<const ulonglong2*>(ws + c * 32 + 2 * i);
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int pr = i + e;  // column pair within the chunk
                                const unsigned long long x2 =
                                    tc::pack2(fmaxf(__uint_as_float(cur[2 * pr]), 0.f),
                                              fmaxf(__uint_as_float(cur[2 * pr + 1]), 0.f));
                                tc::fma2(a2[H >= 32 ? (pr & 3) : (2 * pr) / H], e ? w4.y : w4.x, x2);
                            }
                        }
                        if (H >= 32) {
                            const float2 t = tc::unpack2(tc::add2(tc::add2(a2[0], a2[1 % NA]), tc::add2(a2[2 % NA], a2[3 % NA])));
                            sc[(c * 32) / H] += t.x + t.y;
                        } else {
#pragma unroll
                            for (int e = 0; e < NA; ++e) {
                                const float2 t = tc::unpack2(a2[e]);
                                sc[c * NA + e] = t.x + t.y;
                            }
                        }
                        if (c + 1 < 8) tc::tmem_wait_ld_dep(nxt);
                    }
                    tc::fence_before_sync();
                    mbar_arrive(&acc_empty[g]);

                    const int s_key = j * 128 + tid;  // key position within the batch
                    if (FP8) {
#pragma unroll
                        for (int q = 0; q < C::QG; ++q) sc[q] *= ksc;
                    }
                    if (SCORES) {
#pragma unroll
                        for (int q = 0; q < C::QG; ++q) {
                            const int qi = qg0 + q;
                            if (qi < p.n_q && s_key < p.n_kv)
                                p.scores[(static_cast<size_t>(b) * p.n_q + qi) * p.n_kv + s_key] =
                                    (s_key <= p.q_pos0 + qi) ? sc[q] : -INFINITY;
                        }
                    } else {
                        // every row sees every key of this tile unless the tile reaches the diagonal
                        const bool full_tile = (j * 128 + 127 <= pos0) && (qlast == C::QG);
#pragma unroll
                        for (int q = 0; q < C::QG; ++q) {
                            const bool valid = full_tile | ((q < qlast) & (s_key <= pos0 + q));
                            // admit iff the score ranks above the row's k-th candidate (set by the last prune)
                            const uint32_t key = score_key(sc[q]);
                            const uint2 th = *reinterpret_cast<const uint2*>(&st[q].thr_key);  // (key, idx)
                            const bool adm = valid & ((key > th.x) | ((key == th.x) & (s_key < static_cast<int>(th.y))));
                            topk_append_warp(wkey + q * rstride, widx + q * rstride, cnt[q], key, s_key, adm, sub);
                        }
                    }
                }
                if ((j % CHECK) == CHECK - 1 || j == nkt - 1) {
                    if (lane == 0) {
#pragma unroll
                        for (int q = 0; q < C::QG; ++q) st[q].cnt[wq] = cnt[q];
                    }
                    grp.sync();
                    // decisions every thread of the group takes alike (read between two barriers)
                    unsigned long long need = 0ull, soft = 0ull;
#pragma unroll
                    for (int q = 0; q < C::QG; ++q) {
                        int mx = 0, tot = 0;
#pragma unroll
                        for (int ww = 0; ww < 4; ++ww) {
                            mx = max(mx, st[q].cnt[ww]);
                            tot += st[q].cnt[ww];
                        }
                        need |= (mx > room && tot > p.topk) ? (1ull << q) : 0ull;
                        soft |= (mx > soft_room && tot > p.topk) ? (1ull << q) : 0ull;
                        if (mx > sub && tid == 0) raise_status(p.hdr, DSA_STATUS_OVERFLOW, mx);
                    }
                    // Both groups meet here at the same key tile.  A prune holds its group's
                    // accumulator, and the MMA alternates between the two, so a prune in one group
                    // stalls both: rows of the other group that are well on their way to a prune
                    // are pruned in the same stall.  The barrier also orders every read of the
                    // counts above before any prune below.
                    unsigned long long* nb = sNeed + (chk & 1u) * 4;
                    if (tid == 0) nb[2 * g] = need;
                    named_bar_sync(3, 256);
                    const bool stop = (wg_abort[0] | wg_abort[1]) != 0;
                    if (nb[2 * (g ^ 1)] != 0ull) need |= soft;
                    ++chk;
                    if (stop) { ok = false; break; }
                    if (!SCORES && need) {
#pragma unroll 1
                        for (int q = 0; q < C::QG; ++q) {
                            if ((need >> q) & 1ull) {
                                uint32_t* ck = cbase + static_cast<size_t>(q) * 2 * p.cap;
                                grp.prune_fast(&st[q], ck, reinterpret_cast<int*>(ck + p.cap), p.topk, room - 32,
                                               slack, sortbuf);
                            }
                        }
#pragma unroll
                        for (int q = 0; q < C::QG; ++q)
                            if ((need >> q) & 1ull) cnt[q] = st[q].cnt[wq];

                    }
                }
            }
            if (!ok) break;
#pragma unroll 1
            for (int q = 0; q < C::QG && !SCORES; ++q) {
                const int qi = qg0 + q;
                if (qi >= p.n_q) break;
                uint32_t* ck = cbase + static_cast<size_t>(q) * 2 * p.cap;
                grp.finish(&st[q], ck, reinterpret_cast<int*>(ck + p.cap), p.topk,
                           p.idx_out + (static_cast<size_t>(b) * p.n_q + qi) * p.topk, nullptr, sortbuf);
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 9) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, 512);
    }
}

// ----------------------------------------------------------------- host side
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D row-major [rows, cols] tensor of `esz`-byte elements; box = 128 bytes x box_rows.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, int esz, uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esz};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Candidate buffer entries per row: room for the k survivors of a prune plus at
// least 4 tiles of appends (the epilogue checks every 4 key tiles) and slack.
int cand_cap(int topk) {
    int c = 2 * topk + 256;
    if (c < topk + 4 * 128 + 512) c = topk + 4 * 128 + 512;
    c = (c + 127) / 128 * 128;
    if (c > kCandCap) c = kCandCap;
    return c;
}

int grid_for(int n_tiles, int num_sms) { return n_tiles < num_sms ? n_tiles : num_sms; }

int tiles_per_b(int n_q, int H) { return (n_q + 512 / H - 1) / (512 / H); }

template <int H, int D, bool FP8>
cudaError_t launch_t(const void* q, const float* q_scale, const void* k, const float* k_scale, const float* w, int B,
                     int n_q, int q_pos0, int n_kv, int topk, int* idx_out, float* scores_out, void* ws, int num_sms,
                     cudaStream_t stream) {
    using C = IdxCfg<H, D, FP8>;
    CUtensorMap mq, mk;
    if (!make_map(&mq, q, static_cast<uint64_t>(B) * n_q * H, D, C::ESZ, 256) ||
        !make_map(&mk, k, static_cast<uint64_t>(B) * n_kv, D, C::ESZ, 128))
        return cudaErrorInvalidValue;
    IdxParams p;
    p.w = w;
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.B = B;
    p.n_q = n_q;
    p.q_pos0 = q_pos0;
    p.n_kv = n_kv;
    p.topk = topk;
    p.cap = cand_cap(topk);
    p.tiles_per_b = tiles_per_b(n_q, H);
    p.n_tiles = p.tiles_per_b * B;
    p.idx_out = idx_out;
    p.hdr = static_cast<WsHeader*>(ws);
    p.cand = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + kWsHeaderBytes);
    p.scores = scores_out;
    auto kern = scores_out ? indexer_topk_kernel<H, D, FP8, true> : indexer_topk_kernel<H, D, FP8, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = grid_for(p.n_tiles, num_sms);
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, p);
    return cudaGetLastError();
}

}  // namespace

bool indexer_decode_supported(int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int dtype);
size_t indexer_decode_workspace_bytes(int B, int q_pos0, int topk, int num_sms, bool varlen);
cudaError_t launch_indexer_decode(const void* q, const float* q_scale, const void* k, const float* k_scale,
                                  const float* w, int dtype, int B, int q_pos0, int n_kv, int H, int topk,
                                  int* idx_out, void* ws, int num_sms, cudaStream_t stream);

size_t indexer_workspace_bytes(int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int dtype,
                               int num_sms) {
    if (indexer_decode_supported(B, n_q, q_pos0, n_kv, H, d, topk, dtype))
        return indexer_decode_workspace_bytes(B, q_pos0, topk, num_sms, false);
    const int n_tiles = tiles_per_b(n_q, H) * B;
    const int grid = grid_for(n_tiles, num_sms);
    const size_t qg = 256 / H;
    return static_cast<size_t>(grid) * 2 * qg * 2 * cand_cap(topk) * sizeof(uint32_t);
}

cudaError_t launch_indexer(const void* q, const float* q_scale, const void* k, const float* k_scale, const float* w,
                           int dtype, int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int* idx_out,
                           float* scores_out, void* ws, size_t ws_bytes, int num_sms, cudaStream_t stream) {
    (void)ws_bytes;
    // one query per sequence: the split decode kernel (the selection path only)
    if (!scores_out && indexer_decode_supported(B, n_q, q_pos0, n_kv, H, d, topk, dtype))
        return launch_indexer_decode(q, q_scale, k, k_scale, w, dtype, B, q_pos0, n_kv, H, topk, idx_out, ws, num_sms,
                                     stream);
#define DSA_IDX_CASE(HH, DD, F8)                                                                              \
    if (H == HH && d == DD && (dtype == DSA_E4M3) == F8)                                                     \
        return launch_t<HH, DD, F8>(q, q_scale, k, k_scale, w, B, n_q, q_pos0, n_kv, topk, idx_out, scores_out, ws, \
                                    num_sms, stream);
    DSA_IDX_CASE(4, 64, false)
    DSA_IDX_CASE(4, 128, false)
    DSA_IDX_CASE(8, 128, false)
    DSA_IDX_CASE(16, 128, false)
    DSA_IDX_CASE(32, 128, false)
    DSA_IDX_CASE(64, 128, false)
    DSA_IDX_CASE(32, 128, true)
    DSA_IDX_CASE(64, 128, true)
#undef DSA_IDX_CASE
    return cudaErrorNotSupported;
}

}  // namespace dsa
