// dsa_indexer_decode.cu -- the fused indexer + top-k for decode: one query
// per sequence against a long key cache.
//
// Same operation as dsa_indexer.cu (the DSA lightning indexer, [QbitAI]
// §IndexCache; [Term] "dot product + top-k").  With one query row there is
// no query reuse to harvest, so the work is a scan of the key cache at HBM
// speed: the prefill kernel would give each sequence one CTA and pad each
// MMA to 16 queries.  Here:
//   * Each sequence's key range is split over several CTAs (units of
//     (sequence, split)), so B*splits units cover all SMs.
//   * The MMA is 128 keys x H_I heads (N = H_I, one query) and the 512 TMEM
//     columns hold a ring of 512/H_I accumulators, so many key tiles are in
//     flight while the epilogue drains older ones.
//   * A TMA ring of 128 KB streams the keys (4 bf16 or 8 fp8 stages).
//   * Each unit writes its keys' order-preserving score keys to the row's slots
//     and counts their top bits into a histogram (in the shared memory a
//     candidate buffer would take), added to the row's histogram from the
//     unit's own k-th-key bin up; the bin select (dsa_topk_radix.cu) then
//     picks each row's top-k in one pass over its score keys.
//   * The key cache may be paged (serving: fixed-size pages of tokens, a page
//     table per sequence) and sequences may differ in length: each 128-key
//     tile is fetched page by page, keys past a sequence's length are masked,
//     and units past a sequence's last tile score nothing.
#include <cuda.h>

#include "dsa_tc.cuh"
#include "dsa_topk.cuh"

namespace dsa {

size_t bin_topk_hist_bytes(int rows);
size_t bin_topk_scratch_bytes(int rows, int n, int num_sms);
cudaError_t launch_bin_topk(const uint32_t* keys, long long ld, int rows, int n, int k, int* out, void* scratch,
                            WsHeader* hdr, const int* lens, int len_cap, int num_sms, cudaStream_t stream);

template <int H, bool FP8>
struct DecCfg {
    static constexpr int N = H;              // accumulator columns: one query's heads
    static constexpr int NACC = 512 / N;     // accumulators in flight
    static constexpr int ROWB = FP8 ? 128 : 256;  // bytes per key / query-head row (d_I = 128)
    static constexpr int KB = ROWB / 128;         // 128-byte swizzle blocks per row
    static constexpr int KSTEPS = ROWB / 32;      // MMA K-steps of 32 bytes
    static constexpr int BOX_X = FP8 ? 128 : 64;  // elements per 128-byte TMA box row
    static constexpr int STAGES = FP8 ? 8 : 4;    // the same 128 KB of keys in flight either way
    static constexpr int A_STAGE = 128 * ROWB;    // 128 keys
    static constexpr int B_BYTES = N * ROWB;      // the query's H rows
    static constexpr int CAP = kCandCap;       // candidate buffer of the unit's row (shared memory)
    static constexpr int THREADS = 192;        // warps 0-3 epilogue, 4 producer, 5 MMA
    static constexpr int OFF_B = 0;
    static constexpr int OFF_A = OFF_B + ((B_BYTES + 1023) / 1024) * 1024;
    static constexpr int OFF_CK = OFF_A + STAGES * A_STAGE;
    static constexpr int OFF_CI = OFF_CK + CAP * 4;
    static constexpr int OFF_SORT = OFF_CI + CAP * 4;
    static constexpr int OFF_W = OFF_SORT + DSA_TOPK_MAX * 4;
    static constexpr int OFF_SC = OFF_W + 64 * 4;
    static constexpr int OFF_ST = OFF_SC + static_cast<int>(sizeof(TopkGroup<128>::Scratch));
    static constexpr int OFF_BAR = (OFF_ST + static_cast<int>(sizeof(TopkRowState)) + 7) / 8 * 8;
    static constexpr int NBAR = 2 + 2 * STAGES + 2 * NACC;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct DecParams {
    const float* w;
    const float* q_scale;   // [B, H] (e4m3 only): folded into w
    const float* k_scale;   // [B, n_kv] (e4m3 only): multiplies each key's score
    const int* seq_lens;    // [B] cache length of each sequence, or NULL: every sequence has q_pos0 + 1 keys
    const int* page_table;  // [B, max_pages] physical page of each logical page, or NULL: contiguous [B, n_kv]
    int page_size, max_pages, num_pages;
    int B, q_pos0, n_kv, topk, splits, tiles_per_split;
    uint32_t* score_keys;  // [B, q_pos0 + 1] order-preserving score keys (score mode), or NULL
    int* hist;             // score mode: [B, 2^kBinTopkBits] counts of the keys' top bits (zeroed before)
    WsHeader* hdr;
};

template <int H, bool FP8>
__global__ void __launch_bounds__(192, 1)
    indexer_decode_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                          const DecParams p) {
    using C = DecCfg<H, FP8>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sB = smem + C::OFF_B;
    unsigned char* sA = smem + C::OFF_A;
    uint32_t* ckey = reinterpret_cast<uint32_t*>(smem + C::OFF_CK);
    int* sortbuf = reinterpret_cast<int*>(smem + C::OFF_SORT);
    float* ws = reinterpret_cast<float*>(smem + C::OFF_W);
    auto* sc = reinterpret_cast<TopkGroup<128>::Scratch*>(smem + C::OFF_SC);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* kv_full = bars + 2;
    uint64_t* kv_empty = kv_full + C::STAGES;
    uint64_t* acc_full = kv_empty + C::STAGES;
    uint64_t* acc_empty = acc_full + C::NACC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
    int* wg_abort = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);  // written only by the epilogue

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int units = p.B * p.splits;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int a = 0; a < C::NACC; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 128);
        }
        *abort_flag = 0;
        *wg_abort = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        tc::prefetch_tmap(&tmap_q);
        tc::prefetch_tmap(&tmap_k);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // keys of sequence b (its query sits at the last of them); out-of-range lengths are flagged and clamped
    auto seq_len = [&](int b) -> int {
        if (!p.seq_lens) return p.q_pos0 + 1;
        int len = __ldg(p.seq_lens + b);
        // at most the row of score keys (max_seq_len for a paged cache) and the pages it holds
        const int cap = p.page_table ? min(p.max_pages * p.page_size, p.q_pos0 + 1) : p.n_kv;
        if (len < 1 || len > cap) {
            if (threadIdx.x == 0) raise_status(p.hdr, DSA_STATUS_BAD_INDEX, len);
            len = len < 1 ? 1 : cap;
        }
        return len;
    };
    auto unit_range = [&](int u, int& b, int& j0, int& j1, int& len) {
        b = u / p.splits;
        len = seq_len(b);
        const int sp = u % p.splits;
        j0 = sp * p.tiles_per_split;
        j1 = min((len + 127) / 128, j0 + p.tiles_per_split);  // empty when the sequence is shorter
    };

    if (warp == 4) {
        // ================================================== TMA producer
        if (lane == 0) {
            uint32_t it = 0, wt = 0;
            bool ok = true;
            int pend_q = -1;
            const bool withhold = test_withhold_tile(p.hdr);  // timeout test: first key tile never sent
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++wt) {
                int b, j0, j1, len;
                unit_range(u, b, j0, j1, len);
                if (wt > 0 && !mbar_wait(q_empty, (wt - 1) & 1)) { ok = false; break; }
                mbar_arrive_expect_tx(q_full, C::B_BYTES);
                for (int kb = 0; kb < C::KB; ++kb)
                    tc::tma_load_2d(sB + kb * H * 128, &tmap_q, kb * C::BOX_X, b * H, q_full);
                pend_q = static_cast<int>(wt);
                for (int j = j0; j < j1; ++j, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t rr = it / C::STAGES;
                    if (rr > 0 && !mbar_wait(&kv_empty[s], (rr - 1) & 1)) { ok = false; break; }
                    if (withhold && it == 0) continue;  // nothing issued: the waits on this stage run out
                    mbar_arrive_expect_tx(&kv_full[s], C::A_STAGE);
                    if (FP8 || !p.page_table) {  // (the fp8 form is built for contiguous caches only)
                        for (int kb = 0; kb < C::KB; ++kb)
                            tc::tma_load_2d(sA + s * C::A_STAGE + kb * 128 * 128, &tmap_k, kb * C::BOX_X,
                                            b * p.n_kv + j * 128, &kv_full[s]);
                    } else {
                        // the tile's 128 keys page by page (rows = pieces of min(page, 128) keys; the
                        // pieces start at 1024-byte multiples, so the 128-byte swizzle lines up)
                        const int piece = min(p.page_size, 128);
                        const int used = (len + p.page_size - 1) / p.page_size;  // pages the sequence holds
                        for (int r0 = 0; r0 < 128; r0 += piece) {
                            const int tok = j * 128 + r0;
                            const int lp = tok / p.page_size;
                            int pg = lp < used ? __ldg(p.page_table + static_cast<size_t>(b) * p.max_pages + lp) : 0;
                            if (pg < 0 || pg >= p.num_pages) pg = 0;  // keys there are masked anyway
                            const int row = pg * p.page_size + tok % p.page_size;
                            for (int kb = 0; kb < 2; ++kb)
                                tc::tma_load_2d(sA + s * C::A_STAGE + kb * 128 * 128 + r0 * 128, &tmap_k, kb * 64,
                                                row, &kv_full[s]);
                        }
                    }
                    if (*reinterpret_cast<volatile int*>(abort_flag)) { ok = false; ++it; break; }
                }
            }
            if (!ok) {
                raise_status(p.hdr, DSA_STATUS_TIMEOUT, 0x2d01);
                atomicExch(abort_flag, 1);
            }
            if (pend_q >= 0) mbar_wait(q_full, pend_q & 1);
            for (uint32_t k2 = (it > C::STAGES ? it - C::STAGES : 0); k2 < it; ++k2)
                mbar_wait(&kv_full[k2 % C::STAGES], (k2 / C::STAGES) & 1);
        }
    } else if (warp == 5) {
        // ================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = FP8 ? tc::make_idesc(0, 0, 128, C::N) : tc::make_idesc(1, 1, 128, C::N);
            uint32_t it = 0, wt = 0, ua = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++wt) {
                int b, j0, j1, len;
                unit_range(u, b, j0, j1, len);
                (void)b;
                if (!mbar_wait(q_full, wt & 1)) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t b0 = smem_u32(sB);
                for (int j = j0; j < j1; ++j, ++it, ++ua) {
                    const int s = it % C::STAGES;
                    const int a = ua % C::NACC;
                    if (!mbar_wait(&kv_full[s], (it / C::STAGES) & 1)) { ok = false; break; }
                    if (ua >= C::NACC && !mbar_wait(&acc_empty[a], ((ua / C::NACC) - 1) & 1)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t a0 = smem_u32(sA + s * C::A_STAGE);
#pragma unroll
                    for (int ks = 0; ks < C::KSTEPS; ++ks) {
                        const uint64_t ad = tc::make_sdesc_sw128(a0 + (ks >> 2) * (128 * 128) + (ks & 3) * 32);
                        const uint64_t bd = tc::make_sdesc_sw128(b0 + (ks >> 2) * (H * 128) + (ks & 3) * 32);
                        if (FP8)
                            tc::mma_f8(tmem_base + a * C::N, ad, bd, idesc, ks > 0);
                        else
                            tc::mma_f16(tmem_base + a * C::N, ad, bd, idesc, ks > 0);
                    }
                    tc::mma_commit(&acc_full[a]);
                    tc::mma_commit(&kv_empty[s]);
                    if (*reinterpret_cast<volatile int*>(abort_flag)) { ok = false; break; }
                }
                tc::mma_commit(q_empty);
            }
            if (!ok) {
                raise_status(p.hdr, DSA_STATUS_TIMEOUT, 0x2d02);
                atomicExch(abort_flag, 1);
            }
        }
    } else {
        // ================================================== epilogue (warps 0-3)
        const int tid = threadIdx.x;  // key lane
        TopkGroup<128> grp{tid, 1, sc, C::CAP};  // its named barrier for the four epilogue warps
        constexpr int CHECK = 4;                 // tiles between looks at the abort word
        const uint32_t tlane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        uint32_t ua = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int b, j0, j1, len;
            unit_range(u, b, j0, j1, len);
            if (tid < H) {  // head weights (fp8: folded with the query's per-head scale)
                float wv = p.w[static_cast<size_t>(b) * H + tid];
                if (FP8) wv *= p.q_scale[static_cast<size_t>(b) * H + tid];
                ws[tid] = wv;
            }
            // the unit's histogram of its score keys' top bits lives where candidate buffers would
            int* shist = reinterpret_cast<int*>(ckey);  // 2^kBinTopkBits counts in the ckey + cidx region
            for (int i = tid; i < (1 << kBinTopkBits); i += 128) shist[i] = 0;
            grp.sync();
            for (int j = j0; j < j1; ++j, ++ua) {
                const int a = ua % C::NACC;
                const int s_key = j * 128 + tid;
                // fp8: this key's scale, read before the wait so its latency hides behind it
                const float ksc = (FP8 && s_key < len) ? __ldg(p.k_scale + static_cast<size_t>(b) * p.n_kv + s_key) : 0.f;
                const bool got = __all_sync(0xffffffffu, mbar_wait(&acc_full[a], (ua / C::NACC) & 1));
                float sc_v = 0.f;
                if (got) {
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < H / 32; ++c) {
                        uint32_t v[32];
                        tc::tmem_ld32(tlane + a * C::N + c * 32, v);
                        tc::tmem_wait_ld_dep(v);
                        unsigned long long a2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const unsigned long long w2 = *reinterpret_cast<const unsigned long long*>(ws + c * 32 + 2 * i);
                            tc::fma2(a2[i & 3], w2,
                                     tc::pack2(fmaxf(__uint_as_float(v[2 * i]), 0.f),
                                               fmaxf(__uint_as_float(v[2 * i + 1]), 0.f)));
                        }
                        const float2 t = tc::unpack2(tc::add2(tc::add2(a2[0], a2[1]), tc::add2(a2[2], a2[3])));
                        sc_v += t.x + t.y;
                    }
                    tc::fence_before_sync();
                    mbar_arrive(&acc_empty[a]);
                } else if (lane == 0) {
                    raise_status(p.hdr, DSA_STATUS_TIMEOUT, 0x2d03);
                    atomicExch(abort_flag, 1);
                    *wg_abort = 1;
                }
                if (FP8) sc_v *= ksc;
                const uint32_t key = score_key(sc_v);
                // the row's keys go to memory and into the histogram of their top bits; the bin
                // select picks the top-k
                const bool v = got && s_key < len;
                if (v) {
                    p.score_keys[static_cast<size_t>(b) * (p.q_pos0 + 1) + s_key] = key;
                    atomicAdd(&shist[key >> (32 - kBinTopkBits)], 1);
                }
                if (((j - j0) % CHECK) == CHECK - 1 || j == j1 - 1) {
                    grp.sync();
                    const bool stop = *wg_abort != 0;  // read between two barriers: uniform
                    grp.sync();
                    if (stop) { ok = false; break; }
                }
            }
            if (!ok) break;
            {
                grp.sync();  // every key of the unit is counted
                // Only the bins from this unit's own k-th key up go to the row's histogram: the unit
                // alone holds k keys at or above that bin, so the row's k-th key lies there too, and
                // every bin the row's threshold search looks at still gets all its counts.
                constexpr int NB = 1 << kBinTopkBits, PB = NB / 128;
                int cs = 0;
                for (int j = 0; j < PB; ++j) cs += shist[tid * PB + j];
                int suf = cs;  // keys in bins >= tid * PB, first within the warp
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_down_sync(0xffffffffu, suf, off);
                    if (lane + off < 32) suf += o;
                }
                if (lane == 0) sortbuf[warp] = suf;
                if (tid == 0) sortbuf[4] = 0;
                grp.sync();
                for (int ww = warp + 1; ww < 4; ++ww) suf += sortbuf[ww];
                if (suf >= p.topk && suf - cs < p.topk) {
                    int acc = suf - cs, T = tid * PB;
                    for (int j = PB - 1; j >= 0; --j) {
                        acc += shist[tid * PB + j];
                        if (acc >= p.topk) {
                            T = tid * PB + j;
                            break;
                        }
                    }
                    sortbuf[4] = T;
                }
                grp.sync();
                const int t_lo = sortbuf[4];
                int* gh = p.hist + static_cast<size_t>(b) * NB;
                for (int i = t_lo + tid; i < NB; i += 128) {
                    const int c = shist[i];
                    if (c) atomicAdd(gh + i, c);
                }
                grp.sync();  // before the next unit clears it
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, 512);
    }
}

// ----------------------------------------------------------------- host side
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map_dec(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows, bool fp8) {
    // [rows, 128] bf16 or e4m3, 128-byte swizzled boxes of 128 bytes x box_rows
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {fp8 ? 128u : 256u};
    cuuint32_t box[2] = {fp8 ? 128u : 64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Key-range splits per sequence: about `per_sm` units per SM (per_sm_for: 4 when every sequence has the
// same length; more when lengths differ, so that uneven units still balance), at least 8 key
// tiles a unit.
int dec_splits(int B, int nkt, int num_sms, int per_sm) {
    int s = (per_sm * num_sms + B - 1) / B;
    if (s > nkt / 8) s = nkt / 8;  // keep at least 8 key tiles per unit
    if (s < 1) s = 1;
    return s;
}

// Units per SM: more when lengths differ (uneven units balance better); for a few long
// sequences more units per row would add more unit histograms into the same row's bins.
int per_sm_for(int B, bool varlen) {
    if (varlen) return 6;
    return B >= 32 ? 4 : 2;
}

// Cache geometry of a decode launch.  Contiguous: k [B, n_kv, d], every sequence q_pos0 + 1 keys.
// Paged: k [num_pages * page_size, d], page_table [B, max_pages], seq_lens [B] (device), at most
// max_len keys a sequence (host bound that sizes the split).
struct DecCache {
    const int* seq_lens;
    const int* page_table;
    int page_size, max_pages, num_pages, max_len;
};

template <int H, bool FP8>
cudaError_t launch_dec_t(const void* q, const float* q_scale, const void* k, const float* k_scale, const float* w,
                         int B, int q_pos0, int n_kv, int topk, const DecCache& pc, int* idx_out, void* ws,
                         int num_sms, cudaStream_t stream) {
    using C = DecCfg<H, FP8>;
    CUtensorMap mq, mk;
    const bool paged = pc.page_table != nullptr;
    if (FP8 && paged) return cudaErrorNotSupported;
    const uint64_t krows = paged ? static_cast<uint64_t>(pc.num_pages) * pc.page_size : static_cast<uint64_t>(B) * n_kv;
    if (!make_map_dec(&mq, q, static_cast<uint64_t>(B) * H, H, FP8) ||
        !make_map_dec(&mk, k, krows, paged ? static_cast<uint32_t>(pc.page_size < 128 ? pc.page_size : 128) : 128,
                      FP8))
        return cudaErrorInvalidValue;
    const int max_len = pc.seq_lens ? pc.max_len : q_pos0 + 1;
    const int nkt = (max_len + 127) / 128;
    DecParams p;
    p.w = w;
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.seq_lens = pc.seq_lens;
    p.page_table = pc.page_table;
    p.page_size = pc.page_size;
    p.max_pages = pc.max_pages;
    p.num_pages = pc.num_pages;
    p.B = B;
    p.q_pos0 = q_pos0;
    p.n_kv = n_kv;
    p.topk = topk;
    p.splits = dec_splits(B, nkt, num_sms, per_sm_for(B, pc.seq_lens != nullptr));
    p.tiles_per_split = (nkt + p.splits - 1) / p.splits;
    p.splits = (nkt + p.tiles_per_split - 1) / p.tiles_per_split;  // no empty units
    p.hdr = static_cast<WsHeader*>(ws);
    unsigned char* scratch = static_cast<unsigned char*>(ws) + kWsHeaderBytes;
    // every row's score keys (max_len of them per row) and their histogram, then the bin select
    const size_t keys_bytes = (static_cast<size_t>(B) * max_len * 4 + 255) / 256 * 256;
    p.score_keys = reinterpret_cast<uint32_t*>(scratch);
    p.hist = reinterpret_cast<int*>(scratch + keys_bytes);
    auto kern = indexer_decode_kernel<H, FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.hist, 0, bin_topk_hist_bytes(B), stream)) != cudaSuccess) return e;
    const int units = B * p.splits;
    kern<<<units < num_sms ? units : num_sms, C::THREADS, C::SMEM, stream>>>(mq, mk, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // variable lengths: the select reads each row's length, clamped as the kernel clamped it
    const int len_cap = paged ? (pc.max_pages * pc.page_size < max_len ? pc.max_pages * pc.page_size : max_len)
                              : max_len;
    return launch_bin_topk(p.score_keys, max_len, B, max_len, topk, idx_out, scratch + keys_bytes, p.hdr,
                           pc.seq_lens, len_cap, num_sms, stream);
}

}  // namespace

bool indexer_decode_supported(int B, int n_q, int q_pos0, int n_kv, int H, int d, int topk, int dtype) {
    (void)B;
    (void)n_kv;
    (void)topk;
    return n_q == 1 && d == 128 && (dtype == DSA_BF16 || dtype == DSA_E4M3) && (H == 32 || H == 64) &&
           q_pos0 + 1 >= 8 * 128;
}

size_t indexer_decode_workspace_bytes(int B, int q_pos0, int topk, int num_sms, bool varlen) {
    // the rows' score keys (q_pos0 + 1 per row; for variable lengths q_pos0 = the longest - 1),
    // then the bin select's state
    (void)topk;
    (void)varlen;
    const size_t keys_bytes = (static_cast<size_t>(B) * (q_pos0 + 1) * 4 + 255) / 256 * 256;
    return keys_bytes + bin_topk_scratch_bytes(B, q_pos0 + 1, num_sms);
}

cudaError_t launch_indexer_decode(const void* q, const float* q_scale, const void* k, const float* k_scale,
                                  const float* w, int dtype, int B, int q_pos0, int n_kv, int H, int topk,
                                  int* idx_out, void* ws, int num_sms, cudaStream_t stream) {
    const DecCache none = {nullptr, nullptr, 0, 0, 0, 0};
    const bool f8 = dtype == DSA_E4M3;
#define DSA_DEC_CASE(HH, F8)                                                                                   \
    if (H == HH && f8 == F8)                                                                                   \
        return launch_dec_t<HH, F8>(q, q_scale, k, k_scale, w, B, q_pos0, n_kv, topk, none, idx_out, ws, num_sms, \
                                    stream);
    DSA_DEC_CASE(32, false)
    DSA_DEC_CASE(64, false)
    DSA_DEC_CASE(32, true)
    DSA_DEC_CASE(64, true)
#undef DSA_DEC_CASE
    return cudaErrorNotSupported;
}

cudaError_t launch_indexer_decode_paged(const void* q, const void* k_pages, const int* page_table, const int* seq_lens,
                                        const float* w, int B, int max_len, int page_size, int num_pages,
                                        int max_pages, int H, int topk, int* idx_out, void* ws, int num_sms,
                                        cudaStream_t stream) {
    const DecCache pc = {seq_lens, page_table, page_size, max_pages, num_pages, max_len};
    if (H == 32)
        return launch_dec_t<32, false>(q, nullptr, k_pages, nullptr, w, B, max_len - 1, 0, topk, pc, idx_out, ws,
                                       num_sms, stream);
    if (H == 64)
        return launch_dec_t<64, false>(q, nullptr, k_pages, nullptr, w, B, max_len - 1, 0, topk, pc, idx_out, ws,
                                       num_sms, stream);
    return cudaErrorNotSupported;
}

}  // namespace dsa
