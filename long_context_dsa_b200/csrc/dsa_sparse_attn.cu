// dsa_sparse_attn.cu -- attention over each query's selected tokens (K3).
//
// [Explainer] §稀疏注意力的隐性开销: every token attends only to its top-k
// history tokens; §IndexShare 的共享机制: S layers keep their own attention
// weights, so each layer runs this kernel with its own Q/K/V.
//
// Design (B200): the work is a gather -- every (query, KV head) reads k
// rows of K and V picked by the index cache -- so it is bound by memory,
// not by math.
//   * The unit of work is one (query row, KV head).  Every warp runs its own
//     pipeline over units: it gathers its head's K and V slices (d bf16
//     each, contiguous in the token-major layout) for a chunk of selected
//     tokens with 16-byte cp.async into a private multi-stage ring, and
//     computes on the oldest stage while the younger ones are in flight.
//     Padding entries (-1) become zero-filled copies that read nothing.
//     Indices are read two chunks ahead of their gather and turned into row
//     offsets one chunk ahead, so neither the index load nor a shared
//     producer sits on the critical path.
//   * Online softmax with warp-level bf16 tensor-core MMAs (m16n8k16):
//     S^T = K_chunk Q^T puts keys on M and the GQA group's query heads on N
//     (8 columns: no padding at G = 8); O^T += V^T P puts d on M.  P moves
//     from the S^T accumulator layout into the B-operand layout with
//     movmatrix and is split into bf16 hi + lo parts (two MMAs) so the
//     weights keep ~16 bits.
//   * Ring rows are packed at 2*d bytes with their 16-byte segments XOR-
//     swizzled by (row & 7): every ldmatrix is conflict-free and 14 warps
//     (16-key chunks, 2 stages each) fit in shared memory at d = 128.  On
//     B200 the number of warps in flight set the speed far more than the
//     stages per warp did.
#include <cfloat>
#include <climits>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dsa_common.cuh"

namespace dsa {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// 16-byte async copy global -> shared; src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// SWZ: rows packed at 2*d bytes with their 16-byte segments XOR-swizzled by
// (row & 7) instead of padded, which fits more warps in shared memory.
template <int D, int CHUNK, int STAGES, int WARPS, bool SWZ = false>
struct AttnCfg {
    static constexpr int RS = SWZ ? D * 2 : D * 2 + 16;    // ring row stride (bytes)
    static constexpr int STAGE_BYTES = 2 * CHUNK * RS;     // K rows then V rows
    static constexpr int WARP_BYTES = STAGES * STAGE_BYTES + STAGES * CHUNK * 4;  // + staged indices
    static constexpr int SEGS = D * 2 / 16;                // 16-byte segments per row slice
    static constexpr int KEYS_PER_INSN = 32 / SEGS;        // rows one warp-wide cp.async covers
    static constexpr size_t SMEM = static_cast<size_t>(WARPS) * WARP_BYTES;
    static_assert(CHUNK % 16 == 0 && CHUNK <= 32, "chunk of whole 16-key MMA tiles, one index per lane");
    static_assert(32 % SEGS == 0, "row slice splits evenly over the warp");
    // byte offset of 16-byte segment `sg` of ring row `r`
    __device__ static __forceinline__ uint32_t at(int r, int sg) {
        return static_cast<uint32_t>(r * RS + ((SWZ ? (sg ^ (r & 7)) : sg) << 4));
    }
};

// Compile-time switches, so the plain path carries none of the bookkeeping of the others:
// SPLIT: units cut into index ranges (few rows, e.g. decode); PAGED: K/V in a page pool;
// SHARED: query rows share index rows; OFF32: every row of a sequence's K (and V) lies within
// 2 GB of its first, so row offsets are 32-bit (contiguous caches only).
template <int D, int CHUNK, int STAGES, int WARPS, bool SWZ, bool QK_SPLIT, bool OUT_BF16, bool SPLIT, bool PAGED,
          bool SHARED, bool OFF32 = false>
__global__ void __launch_bounds__(WARPS * 32)
    sparse_attn_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                       const __nv_bfloat16* __restrict__ V, const int* __restrict__ idx, int B, int n_q,
                       int n_kv, int Hq, int Hkv, int topk, float scale_log2, void* __restrict__ O,
                       int splits, int chunks_per_split, float* __restrict__ part, IdxShare share,
                       KvPages pg, WsHeader* hdr) {
    using C = AttnCfg<D, CHUNK, STAGES, WARPS, SWZ>;
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* ring = smem + warp * C::WARP_BYTES;
    int* sidx = reinterpret_cast<int*>(ring + STAGES * C::STAGE_BYTES);
    const uint32_t ring_s = smem_u32(ring);

    const int G = Hq / Hkv;
    // work items: (query row, KV head) units, each cut into `splits` ranges of chunks; with
    // splits > 1 a warp writes its range's softmax state to `part` and attn_merge_kernel combines
    const long long units = static_cast<long long>(B) * n_q * Hkv;
    const long long items = SPLIT ? units * splits : units;
    const int nchunks = (topk + CHUNK - 1) / CHUNK;
    const size_t tok_stride = static_cast<size_t>(Hkv) * D;  // elements per token row of K / V

    const int qn = lane >> 2;        // query head (N column) this lane loads for Q; key row in C tiles
    const int hc = 2 * (lane & 3);   // first of the two head columns this lane owns in C tiles
    const int lrow = lane & 7, lq = lane >> 3;
    const int k_key_off = ((lq & 1) ? 8 : 0) + lrow, k_d_off = (lq >= 2) ? 8 : 0;   // K: non-trans A
    const int v_key_off = ((lq >= 2) ? 8 : 0) + lrow, v_d_off = (lq & 1) ? 8 : 0;  // V: trans A
    const int seg = lane % C::SEGS, sub = lane / C::SEGS;  // copy: segment within a row, row within an insn

    for (long long it = static_cast<long long>(blockIdx.x) * WARPS + warp; it < items;
         it += static_cast<long long>(gridDim.x) * WARPS) {
        const long long u = SPLIT ? it / splits : it;
        const int sp = SPLIT ? static_cast<int>(it % splits) : 0;
        const int c0 = SPLIT ? sp * chunks_per_split : 0;
        const int c1 = SPLIT ? min(nchunks, c0 + chunks_per_split) : nchunks;
        // unsplit units run KV head by KV head (all rows of head 0, then head 1, ...): the rows in
        // flight at once then gather from one head's K/V, which fits in L2 where all heads' do not;
        // split ranges keep (row, head) order, the order their merge reads them in
        const long long nrows = static_cast<long long>(B) * n_q;
        const long long row = SPLIT ? u / Hkv : u % nrows;
        const int g = static_cast<int>(SPLIT ? u % Hkv : u / nrows);
        const long long b = row / n_q;
        const int qi = static_cast<int>(row - b * n_q);
        const int* irow = SHARED ? idx + (b * share.rows(n_q) + qi / share.q_per_idx) * topk : idx + row * topk;
        const int lim = SHARED ? share.limit(qi) : 0;  // shared rows: keys past the query's own position are skipped
        const size_t seq_off = PAGED ? 0 : static_cast<size_t>(b) * n_kv * tok_stride;
        const __nv_bfloat16* kb = K + seq_off + static_cast<size_t>(g) * D;
        const __nv_bfloat16* vb = V + seq_off + static_cast<size_t>(g) * D;
        const int n_valid = PAGED ? min(__ldg(pg.lens + b), pg.max_pages * pg.page_size) : n_kv;
        // OFF32: this lane's 16-byte segment of a row at byte offset 0 (K and V)
        const unsigned char* kseg = reinterpret_cast<const unsigned char*>(kb) + seg * 16;
        const unsigned char* vseg = reinterpret_cast<const unsigned char*>(vb) + seg * 16;

        // Index of key `lane` of chunk c (-1 past the end), read two chunks ahead of its gather, then
        // checked and mapped to its cache row one chunk ahead (so a page-table read never waits on
        // the index read it depends on); out-of-range entries are flagged and skipped.
        auto load_raw = [&](int c) -> int {
            const int kk = c * CHUNK + lane;
            return (lane < CHUNK && kk < topk) ? __ldg(irow + kk) : -1;
        };
        auto map_idx = [&](int t) -> int {
            if (t < -1 || t >= n_valid) {
                raise_status(hdr, DSA_STATUS_BAD_INDEX, t);
                t = -1;
            }
            if (SHARED && t > lim) t = -1;
            if (PAGED && t >= 0) {
                const int page = __ldg(pg.table + static_cast<size_t>(b) * pg.max_pages + pg.page_of(t));
                if (page < 0 || page >= pg.num_pages) {
                    raise_status(hdr, DSA_STATUS_BAD_INDEX, page);
                    t = -1;
                } else {
                    t = page * pg.page_size + pg.in_page(t);
                }
            }
            return t;
        };
        // gather chunk c's K and V slices into stage c % STAGES (always commits one group)
        auto issue = [&](int c, int tsel) {
            if (c < c1) {
                const int s = static_cast<int>(static_cast<unsigned>(SPLIT ? c - c0 : c) % STAGES);
                if (lane < CHUNK) sidx[s * CHUNK + lane] = tsel;
                const uint32_t kst = ring_s + s * C::STAGE_BYTES;
                const uint32_t vst = kst + CHUNK * C::RS;
                if constexpr (OFF32) {
                    // the lane holding a key turns it into its row's byte offset once (padding: the
                    // sign bit alone); the copying lanes shuffle that word in and mask it
                    const int w = tsel >= 0 ? tsel * static_cast<int>(tok_stride * 2) : INT_MIN;
#pragma unroll
                    for (int i = 0; i < CHUNK / C::KEYS_PER_INSN; ++i) {
                        const int key = i * C::KEYS_PER_INSN + sub;
                        const int wk = __shfl_sync(0xffffffffu, w, key);
                        const uint32_t nb = wk >= 0 ? 16u : 0u;
                        const uint32_t o = static_cast<uint32_t>(wk) & 0x7fffffffu;
                        cp_async16(kst + C::at(key, seg), kseg + o, nb);
                        cp_async16(vst + C::at(key, seg), vseg + o, nb);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < CHUNK / C::KEYS_PER_INSN; ++i) {
                        const int key = i * C::KEYS_PER_INSN + sub;
                        const int t = __shfl_sync(0xffffffffu, tsel, key);
                        const uint32_t nb = t >= 0 ? 16u : 0u;
                        const size_t off = static_cast<size_t>(t >= 0 ? t : 0) * tok_stride + seg * 8;
                        cp_async16(kst + C::at(key, seg), kb + off, nb);
                        cp_async16(vst + C::at(key, seg), vb + off, nb);
                    }
                }
            }
            cp_async_commit();
        };

        // Q^T fragments: B[k=d][n=head]
        uint32_t qf[D / 16][2];
        {
            const bool live = qn < G;
            const __nv_bfloat16* qp = Q + (static_cast<size_t>(row) * Hq + g * G + (live ? qn : 0)) * D + hc;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qf[ks][0] = live ? __ldg(reinterpret_cast<const uint32_t*>(qp + ks * 16)) : 0u;
                qf[ks][1] = live ? __ldg(reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8)) : 0u;
            }
        }
        float o[D / 16][4];
#pragma unroll
        for (int i = 0; i < D / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        // running max starts at -FLT_MAX, not -inf: it stays finite, so the rescale and the weights
        // need no guard (a masked score is -inf and weighs exp2(-inf) = 0; before any valid key
        // the factor is exp2(0) = 1), and a range that saw no key reports -FLT_MAX to the merge,
        // where it weighs 0 beside any range that did
        float mrun[2] = {-FLT_MAX, -FLT_MAX}, lrun[2] = {0.f, 0.f};

        // prologue: stages 0 .. STAGES-2 in flight, the next chunk's rows and the one after's
        // indices in registers
        __syncwarp();
#pragma unroll
        for (int c = 0; c < STAGES - 1; ++c) issue(c0 + c, map_idx(load_raw(c0 + c)));
        int t_next = map_idx(load_raw(c0 + STAGES - 1));
        int r_next = load_raw(c0 + STAGES);

        for (int c = c0; c < c1; ++c) {
            issue(c + STAGES - 1, t_next);
            t_next = map_idx(r_next);
            r_next = load_raw(c + STAGES + 1);
            cp_async_wait<STAGES - 1>();
            __syncwarp();
            const int s = static_cast<int>(static_cast<unsigned>(SPLIT ? c - c0 : c) % STAGES);
            const uint32_t kst = ring_s + s * C::STAGE_BYTES;
            const uint32_t vst = kst + CHUNK * C::RS;
            const int* si = sidx + s * CHUNK;
            constexpr int MT = CHUNK / 16;
            // ---- S^T = K Q^T
            float sacc[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                float s2[4] = {0.f, 0.f, 0.f, 0.f};  // second accumulation chain (QK_SPLIT)
                sacc[mt][0] = sacc[mt][1] = sacc[mt][2] = sacc[mt][3] = 0.f;
                const int krow = mt * 16 + k_key_off;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(kst + C::at(krow, 2 * ks + k_d_off / 8), a0, a1, a2, a3);
                    if (QK_SPLIT && (ks & 1))
                        mma_bf16(s2, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                    else
                        mma_bf16(sacc[mt], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                }
                if (QK_SPLIT) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc[mt][e] += s2[e];
                }
            }
            // ---- mask, scale, online softmax
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const bool v0 = si[mt * 16 + qn] >= 0;
                const bool v1 = si[mt * 16 + qn + 8] >= 0;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    sacc[mt][j] = v0 ? sacc[mt][j] * scale_log2 : -INFINITY;
                    sacc[mt][2 + j] = v1 ? sacc[mt][2 + j] * scale_log2 : -INFINITY;
                    mx[j] = fmaxf(mx[j], fmaxf(sacc[mt][j], sacc[mt][2 + j]));
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], off));
            }
            float alpha[2], mnew[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                mnew[j] = fmaxf(mrun[j], mx[j]);
                alpha[j] = exp2f(mrun[j] - mnew[j]);
                mrun[j] = mnew[j];
                lrun[j] *= alpha[j];
            }
            uint32_t phi[MT][2], plo[MT][2];  // [k-step][key rows 0-7 / 8-15]
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                float p[4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    p[j] = exp2f(sacc[mt][j] - mnew[j]);
                    p[2 + j] = exp2f(sacc[mt][2 + j] - mnew[j]);
                    lrun[j] += p[j] + p[2 + j];
                }
                const uint32_t h01 = pack_bf16(p[0], p[1]);
                const uint32_t h23 = pack_bf16(p[2], p[3]);
                const __nv_bfloat162 hh01 = *reinterpret_cast<const __nv_bfloat162*>(&h01);
                const __nv_bfloat162 hh23 = *reinterpret_cast<const __nv_bfloat162*>(&h23);
                const uint32_t l01 = pack_bf16(p[0] - __low2float(hh01), p[1] - __high2float(hh01));
                const uint32_t l23 = pack_bf16(p[2] - __low2float(hh23), p[3] - __high2float(hh23));
                phi[mt][0] = movm_t(h01);
                phi[mt][1] = movm_t(h23);
                plo[mt][0] = movm_t(l01);
                plo[mt][1] = movm_t(l23);
            }
            // ---- O^T = alpha * O^T + V^T P; the rescale is skipped (exactly: alpha == 1) while no
            // head's running max moved
            if (__any_sync(0xffffffffu, (alpha[0] != 1.f) | (alpha[1] != 1.f))) {
#pragma unroll
                for (int dt = 0; dt < D / 16; ++dt) {
                    o[dt][0] *= alpha[0];
                    o[dt][1] *= alpha[1];
                    o[dt][2] *= alpha[0];
                    o[dt][3] *= alpha[1];
                }
            }
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
#pragma unroll
                for (int ks = 0; ks < MT; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(vst + C::at(ks * 16 + v_key_off, 2 * dt + v_d_off / 8), a0, a1, a2, a3);
                    mma_bf16(o[dt], a0, a1, a2, a3, phi[ks][0], phi[ks][1]);
                    mma_bf16(o[dt], a0, a1, a2, a3, plo[ks][0], plo[ks][1]);
                }
            }
            __syncwarp();  // every lane is done with stage s before it is refilled
        }
        cp_async_wait<0>();  // retire the trailing (empty) groups before the ring is reused
        // ---- finalize: row sums across the 8 lanes sharing a head column
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) lrun[j] += __shfl_xor_sync(0xffffffffu, lrun[j], off);
        }
        if (SPLIT) {
            // this range's state per head: unnormalised O, running max (log2 units), sum
            float* pb = part + static_cast<size_t>(it) * G * (D + 2);
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                const int d0 = dt * 16 + qn;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = hc + j;
                    if (h < G) {
                        pb[h * (D + 2) + d0] = o[dt][j];
                        pb[h * (D + 2) + d0 + 8] = o[dt][2 + j];
                    }
                }
            }
            if (qn == 0) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = hc + j;
                    if (h < G) {
                        pb[h * (D + 2) + D] = mrun[j];
                        pb[h * (D + 2) + D + 1] = lrun[j];
                    }
                }
            }
            continue;
        }
        const float inv0 = lrun[0] > 0.f ? 1.f / lrun[0] : 0.f;
        const float inv1 = lrun[1] > 0.f ? 1.f / lrun[1] : 0.f;
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
            const int d0 = dt * 16 + qn;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = hc + j;
                if (h < G) {
                    const float inv = j ? inv1 : inv0;
                    const size_t ob = (static_cast<size_t>(row) * Hq + g * G + h) * D;
                    if (OUT_BF16) {
                        __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(O) + ob;
                        op[d0] = __float2bfloat16_rn(o[dt][j] * inv);
                        op[d0 + 8] = __float2bfloat16_rn(o[dt][2 + j] * inv);
                    } else {
                        float* op = reinterpret_cast<float*>(O) + ob;
                        op[d0] = o[dt][j] * inv;
                        op[d0 + 8] = o[dt][2 + j] * inv;
                    }
                }
            }
        }
    }
}

// Combine the split ranges of each (query row, KV head, query head):
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (ranges that saw no
// key have m_s = -inf and drop out).  One block per unit, one warp per query head: lane s
// holds range s's (m, l) (splits <= 32), the weights reach every lane by shuffles, and each
// lane accumulates D/32 output columns with the ranges' loads independent of each other.
template <int D, bool OUT_BF16>
__global__ void attn_merge_kernel(const float* __restrict__ part, int G, int splits, int Hq, int Hkv,
                                  void* __restrict__ O) {
    const long long u = blockIdx.x;  // (row, g)
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (h >= G) return;
    const long long row = u / Hkv;
    const int g = static_cast<int>(u % Hkv);
    const size_t sstride = static_cast<size_t>(G) * (D + 2);
    const float* p0 = part + (static_cast<size_t>(u) * splits * G + h) * (D + 2);
    const float m = lane < splits ? __ldg(p0 + lane * sstride + D) : -INFINITY;
    const float l = lane < splits ? __ldg(p0 + lane * sstride + D + 1) : 0.f;
    float M = m;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
    float L = f * l;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float acc[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int s2 = 0; s2 < splits; ++s2) {
        const float fs = __shfl_sync(0xffffffffu, f, s2);
#pragma unroll
        for (int i = 0; i < D / 32; ++i) acc[i] += fs * __ldg(p0 + s2 * sstride + i * 32 + lane);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const size_t ob = (static_cast<size_t>(row) * Hq + static_cast<size_t>(g) * G + h) * D;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
        if (OUT_BF16)
            reinterpret_cast<__nv_bfloat16*>(O)[ob + i * 32 + lane] = __float2bfloat16_rn(acc[i] * inv);
        else
            reinterpret_cast<float*>(O)[ob + i * 32 + lane] = acc[i] * inv;
    }
}

// Warps per CTA of the dense configurations (one CTA per SM fits in shared memory).  With fewer
// (row, KV head) units than warps on the GPU (decode), d = 128 runs 32-key chunks over 7 warps:
// fewer, longer steps per warp, measured faster on B200 for 64 sequences x 4 KV heads.
static constexpr int kAttnWarpsD128 = 14;
static constexpr int kAttnWarpsD64 = 16;
static constexpr int kAttnDecodeChunkD128 = 32;
static constexpr int kAttnDecodeWarpsD128 = 7;
// fp8 K/V (d = 128): 3 stages of 16-key chunks over 14 warps
static constexpr int kAttnFp8StagesD128 = 3;
static constexpr int kAttnFp8WarpsD128 = 14;
static constexpr int kAttnFp8StagesD64 = 4;
static constexpr int kAttnFp8WarpsD64 = 16;

static bool attn_decode_shape(long long units, int d, int num_sms) {
    return d == 128 && units < static_cast<long long>(num_sms) * kAttnWarpsD128;
}

// Ranges per unit: 1 when the (row, KV head) units alone give every warp of the GPU (one CTA
// per SM) work.  Otherwise each warp takes work items (unit, range) in turn, so the busiest warp
// handles ceil(units * s / warps) items of ceil(nchunks / s) chunks; the count s (at most 32,
// one lane per range in the merge) that makes this smallest is taken, the smallest such s on
// ties (fewer ranges: fewer pipeline starts, a smaller merge).  Depends only on the shape and
// SM count, so the workspace query and the launch agree.
static int attn_splits(long long units, int nchunks, int warps, int num_sms, int* per) {
    const long long tw = static_cast<long long>(num_sms) * warps;
    int best = 1;
    long long best_cost = -1;
    for (int s = 1; s <= 32 && s <= nchunks && (s == 1 || units < tw); ++s) {
        const int p = (nchunks + s - 1) / s;
        if ((nchunks + p - 1) / p != s) continue;  // this s makes the same ranges as a smaller one
        const long long cost = ((units * s + tw - 1) / tw) * p;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    *per = (nchunks + best - 1) / best;
    return best;
}

template <int D, int CHUNK, int STAGES, int WARPS, bool SWZ = false, bool QK_SPLIT = false>
static cudaError_t launch_attn_t(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                                 const int* idx, int B, int n_q, int n_kv, int Hq, int Hkv, int topk,
                                 float scale, void* O, bool out_bf16, IdxShare share, KvPages pg, WsHeader* hdr,
                                 int num_sms, cudaStream_t stream) {
    using C = AttnCfg<D, CHUNK, STAGES, WARPS, SWZ>;
    const long long units = static_cast<long long>(B) * n_q * Hkv;
    const int nchunks = (topk + CHUNK - 1) / CHUNK;
    int per = nchunks;
    const int splits = attn_splits(units, nchunks, WARPS, num_sms, &per);
    using KernFn = void (*)(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, const int*, int, int, int,
                            int, int, int, float, void*, int, int, float*, IdxShare, KvPages, WsHeader*);
    // (out_bf16, split, paged, shared); paged and shared never combine in the API
#define DSA_K(OB, SP, PG, SH) sparse_attn_kernel<D, CHUNK, STAGES, WARPS, SWZ, QK_SPLIT, OB, SP, PG, SH>
    static const KernFn table[2][2][3] = {
        {{DSA_K(false, false, false, false), DSA_K(false, false, true, false), DSA_K(false, false, false, true)},
         {DSA_K(false, true, false, false), DSA_K(false, true, true, false), DSA_K(false, true, false, true)}},
        {{DSA_K(true, false, false, false), DSA_K(true, false, true, false), DSA_K(true, false, false, true)},
         {DSA_K(true, true, false, false), DSA_K(true, true, true, false), DSA_K(true, true, false, true)}}};
#define DSA_K32(OB, SP) sparse_attn_kernel<D, CHUNK, STAGES, WARPS, SWZ, QK_SPLIT, OB, SP, false, false, true>
    static const KernFn table32[2][2] = {{DSA_K32(false, false), DSA_K32(false, true)},
                                         {DSA_K32(true, false), DSA_K32(true, true)}};
#undef DSA_K32
#undef DSA_K
    const int mode = pg.table ? 1 : (share.q_per_idx > 1 || share.causal) ? 2 : 0;
    // contiguous caches whose per-sequence K (and V) spans under 2 GB take 32-bit row offsets
    const bool off32 = mode == 0 && static_cast<long long>(n_kv) * Hkv * D * 2 <= 0x7fffffffLL;
    KernFn kern = off32 ? table32[out_bf16 ? 1 : 0][splits > 1 ? 1 : 0] : table[out_bf16 ? 1 : 0][splits > 1 ? 1 : 0][mode];
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, WARPS * 32, C::SMEM);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    long long grid = static_cast<long long>(num_sms) * per_sm;
    const long long need = (units * splits + WARPS - 1) / WARPS;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    const float scale_log2 = scale * 1.4426950408889634f;
    float* part = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(hdr) + kWsHeaderBytes);
    kern<<<static_cast<int>(grid), WARPS * 32, C::SMEM, stream>>>(Q, K, V, idx, B, n_q, n_kv, Hq, Hkv, topk,
                                                                   scale_log2, O, splits, per, part, share, pg, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess || splits == 1) return e;
    const int G = Hq / Hkv;
    if (splits > 32) return cudaErrorInvalidValue;  // attn_splits makes at most 32
    if (out_bf16)
        attn_merge_kernel<D, true><<<static_cast<unsigned>(units), G * 32, 0, stream>>>(part, G, splits, Hq, Hkv, O);
    else
        attn_merge_kernel<D, false><<<static_cast<unsigned>(units), G * 32, 0, stream>>>(part, G, splits, Hq, Hkv, O);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// fp8 K/V cache (paged decode).  K and V are stored as OCP E4M3 codes with one fp32 scale per
// (token, KV head): the real row is code x scale.  The gather moves half the bytes of bf16 rows.
//   * Each warp's ring holds the codes (d bytes per row slice) of STAGES 16-key chunks, gathered
//     with cp.async like the bf16 kernel (16-byte segments XOR-swizzled by row); every row's two
//     scales ride along.  Indices are read two chunks ahead, pool rows one chunk ahead.
//   * The MMA fragments come straight from the codes (f16 MMAs; every E4M3 value is an fp16
//     value):  S^T = K Q^T takes each lane's 4 consecutive code bytes of a key row as its A
//     elements, which permutes d inside each 16-wide k-step; Q's fragments are loaded with the
//     same permutation, so the dot products are unchanged.  O^T += V^T P loads the V codes with
//     ldmatrix.trans (pairs of bytes as 16-bit elements), regroups the bytes so each register
//     holds two keys of one d, and widens them; rows of O^T (d) come out interleaved (even d,
//     then odd d, per 16) and are written back in place.
//   * The K scale multiplies the fp32 score.  The V scale goes into the weights instead of the
//     rows: P'[key] = p x vs[key] / vmax with vmax the largest V scale of the range so far, so
//     P' stays in [0, 1] and its fp16 hi + lo parts keep ~22 bits; O^T is held in units of vmax
//     (rescaled when a larger scale arrives) and the V codes widen to fp16 exactly.
// The split rule (and so the workspace) is the bf16 kernel's for the same d.
template <int D, int STAGES, int WARPS>
struct Fp8AttnCfg {
    static constexpr int CHUNK = 16;
    static constexpr int STAGE_BYTES = 2 * CHUNK * D;    // K codes, then V codes (d bytes a row)
    static constexpr int META = STAGES * CHUNK * 12;     // per stage and key: pool row, K scale, V scale
    static constexpr int WARP_BYTES = STAGES * STAGE_BYTES + META;
    static constexpr size_t SMEM = static_cast<size_t>(WARPS) * WARP_BYTES;
    static constexpr int SEG8 = D / 16;                  // 16-byte segments of a code row slice
    static constexpr int KEYS_PER_INSN = 32 / SEG8;
    static_assert(D == 64 || D == 128, "code rows of 4 or 8 segments");
    // byte offset of segment sg of code row r: the 8 rows one ldmatrix (or one quarter of the
    // warp's 4-byte loads) touches land in 8 different 16-byte bank groups
    __device__ static __forceinline__ uint32_t at(int r, int sg) {
        const int f = D == 128 ? (r & 7) : ((r >> 1) & 3);
        return static_cast<uint32_t>(r * D + ((sg ^ f) << 4));
    }
};

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// four E4M3 codes (low byte first) -> bytes 0-1 and bytes 2-3 as two pairs of fp16 values, exactly
// (the word is split into its 16-bit halves in registers, no shift)
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t four, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(four));
}

template <int D, int STAGES, int WARPS, bool OUT_BF16, bool SPLIT>
__global__ void __launch_bounds__(WARPS * 32, 1)
    sparse_attn_fp8_kernel(const __nv_bfloat16* __restrict__ Q, const unsigned char* __restrict__ K8,
                           const float* __restrict__ k_scale, const unsigned char* __restrict__ V8,
                           const float* __restrict__ v_scale, const int* __restrict__ idx, int B, int Hq, int Hkv,
                           int topk, float scale_log2, void* __restrict__ O, int splits, int chunks_per_split,
                           float* __restrict__ part, KvPages pg, WsHeader* hdr) {
    using C = Fp8AttnCfg<D, STAGES, WARPS>;
    constexpr int CHUNK = C::CHUNK;
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* ring = smem + warp * C::WARP_BYTES;
    const uint32_t ring_s = smem_u32(ring);
    int* srow = reinterpret_cast<int*>(ring + STAGES * C::STAGE_BYTES);
    float* sks = reinterpret_cast<float*>(srow + STAGES * CHUNK);
    float* svs = sks + STAGES * CHUNK;

    const int G = Hq / Hkv;
    const long long units = static_cast<long long>(B) * Hkv;  // one query per sequence
    const long long items = SPLIT ? units * splits : units;
    const int nchunks = (topk + CHUNK - 1) / CHUNK;
    const size_t tok_stride = static_cast<size_t>(Hkv) * D;  // bytes per token row of the code pools

    const int qn = lane >> 2;           // key row (S^T) / head column (Q, P) / d pair (V^T) of this lane
    const int c4 = lane & 3;
    const int hc = 2 * c4;              // first of the two head columns this lane owns in C tiles
    const int seg = lane % C::SEG8, sub = lane / C::SEG8;
    // ldmatrix.x4 over K (and .trans over V): matrices (keys 0-7 | keys 8-15) x (segment | + 1)
    const int v_key = ((lane >> 3) & 1) * 8 + (lane & 7), v_seg = lane >> 4;
    const int k_row = v_key, k_sg = v_seg;

    for (long long it = static_cast<long long>(blockIdx.x) * WARPS + warp; it < items;
         it += static_cast<long long>(gridDim.x) * WARPS) {
        const long long u = SPLIT ? it / splits : it;
        const int sp = SPLIT ? static_cast<int>(it % splits) : 0;
        const int c0 = SPLIT ? sp * chunks_per_split : 0;
        const int c1 = SPLIT ? min(nchunks, c0 + chunks_per_split) : nchunks;
        const long long b = u / Hkv;
        const int g = static_cast<int>(u % Hkv);
        const int* irow = idx + b * topk;
        const unsigned char* kb = K8 + static_cast<size_t>(g) * D;
        const unsigned char* vb = V8 + static_cast<size_t>(g) * D;
        const int n_valid = min(__ldg(pg.lens + b), pg.max_pages * pg.page_size);

        // The index of key `lane` of chunk c is read two chunks ahead of its gather and mapped to
        // its pool row (page-table read, checks) one chunk ahead, so neither dependent read sits
        // on the critical path; the row's two scales travel with its codes (cp.async).
        auto load_raw = [&](int c) -> int {
            const int kk = c * CHUNK + lane;
            return (lane < CHUNK && kk < topk) ? __ldg(irow + kk) : -1;
        };
        auto map_row = [&](int t) -> int {  // logical position -> pool row (-1: padding or flagged)
            if (t < -1 || t >= n_valid) {
                raise_status(hdr, DSA_STATUS_BAD_INDEX, t);
                t = -1;
            }
            if (t >= 0) {
                const int page = __ldg(pg.table + static_cast<size_t>(b) * pg.max_pages + pg.page_of(t));
                if (page < 0 || page >= pg.num_pages) {
                    raise_status(hdr, DSA_STATUS_BAD_INDEX, page);
                    t = -1;
                } else {
                    t = page * pg.page_size + pg.in_page(t);
                }
            }
            return t;
        };
        auto issue = [&](int c, int tsel) {
            if (c < c1) {
                const int s = (SPLIT ? c - c0 : c) % STAGES;
                if (lane < CHUNK) {
                    srow[s * CHUNK + lane] = tsel;
                    const size_t so = static_cast<size_t>(tsel >= 0 ? tsel : 0) * Hkv + g;
                    const uint32_t nb = tsel >= 0 ? 4u : 0u;
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(sks + s * CHUNK + lane)),
                                 "l"(k_scale + so), "r"(nb)
                                 : "memory");
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(svs + s * CHUNK + lane)),
                                 "l"(v_scale + so), "r"(nb)
                                 : "memory");
                }
                const uint32_t kst = ring_s + s * C::STAGE_BYTES;
                const uint32_t vst = kst + CHUNK * D;
#pragma unroll
                for (int i = 0; i < CHUNK / C::KEYS_PER_INSN; ++i) {
                    const int key = i * C::KEYS_PER_INSN + sub;
                    const int t = __shfl_sync(0xffffffffu, tsel, key);
                    const uint32_t nb = t >= 0 ? 16u : 0u;
                    const size_t off = static_cast<size_t>(t >= 0 ? t : 0) * tok_stride + seg * 16;
                    cp_async16(kst + C::at(key, seg), kb + off, nb);
                    cp_async16(vst + C::at(key, seg), vb + off, nb);
                }
            }
            cp_async_commit();
        };

        // Q^T fragments in fp16, d permuted like the K fragments: k-step ks takes d = 16 ks + 4 c4
        // + {0,1} (rows 2 c4, 2 c4 + 1 of B) and + {2,3} (rows 2 c4 + 8, 2 c4 + 9)
        uint32_t qf[D / 16][2];
        {
            const bool live = qn < G;
            const __nv_bfloat16* qp = Q + (static_cast<size_t>(b) * Hq + g * G + (live ? qn : 0)) * D + 4 * c4;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint2 raw = live ? __ldg(reinterpret_cast<const uint2*>(qp + ks * 16)) : make_uint2(0u, 0u);
                const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
                const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
                qf[ks][0] = pack_f16(f0.x, f0.y);
                qf[ks][1] = pack_f16(f1.x, f1.y);
            }
        }
        float o[D / 16][4];
#pragma unroll
        for (int i = 0; i < D / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};
        float vmax = 0.f, rvmax = 0.f;  // largest |V scale| of the range so far (O^T is held in its units)

        __syncwarp();
#pragma unroll
        for (int c = 0; c < STAGES - 1; ++c) issue(c0 + c, map_row(load_raw(c0 + c)));
        int t_next = map_row(load_raw(c0 + STAGES - 1));  // pool rows of the next chunk to gather
        int r_next = load_raw(c0 + STAGES);                // raw indices of the one after

        for (int c = c0; c < c1; ++c) {
            issue(c + STAGES - 1, t_next);
            t_next = map_row(r_next);
            r_next = load_raw(c + STAGES + 1);
            cp_async_wait<STAGES - 1>();
            __syncwarp();
            const int s = (SPLIT ? c - c0 : c) % STAGES;
            const uint32_t kst = ring_s + s * C::STAGE_BYTES;
            const uint32_t vst = kst + CHUNK * D;
            const int* si = srow + s * CHUNK;
            const float* ks_ = sks + s * CHUNK;
            const float* vs_ = svs + s * CHUNK;
            // ---- S^T = K Q^T: A rows qn and qn + 8 take code bytes 16 ks + 4 c4 .. + 3; one
            // ldmatrix.x4 (8 rows x 16 bytes per matrix) delivers them for two k-steps
            float sacc[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < D / 16; ks += 2) {
                uint32_t w[4];  // key rows qn / qn + 8 at k-step ks, then at ks + 1
                ldsm_x4(kst + C::at(k_row, ks + k_sg), w[0], w[1], w[2], w[3]);
                uint32_t a[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) e4m3x4_to_f16x2x2(w[i], a[2 * i], a[2 * i + 1]);
                // A fragment (a0, a1, a2, a3) = (row qn bytes 0-1, row qn + 8 bytes 0-1, row qn bytes 2-3, ...)
                mma_f16(sacc, a[0], a[2], a[1], a[3], qf[ks][0], qf[ks][1]);
                mma_f16(s2, a[4], a[6], a[5], a[7], qf[ks + 1][0], qf[ks + 1][1]);
            }
            // ---- mask, K scale, softmax scale, online softmax
            const bool v0 = si[qn] >= 0, v1 = si[qn + 8] >= 0;
            const float f0 = ks_[qn] * scale_log2, f1 = ks_[qn + 8] * scale_log2;
            float mx[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                sacc[j] = v0 ? (sacc[j] + s2[j]) * f0 : -INFINITY;
                sacc[2 + j] = v1 ? (sacc[2 + j] + s2[2 + j]) * f1 : -INFINITY;
                mx[j] = fmaxf(sacc[j], sacc[2 + j]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], off));
            }
            // V scales fold into the weights: P'[key] = p * vs[key] / vmax, in [0, 1], so its fp16
            // hi + lo parts keep ~22 bits; when a chunk brings a larger scale, O^T (held in units
            // of vmax) is rescaled like the running max's alpha.
            const float vq0 = vs_[qn], vq1 = vs_[qn + 8];
            float cmax = fmaxf(fabsf(vq0), fabsf(vq1));
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
            float beta = 1.f;
            if (cmax > vmax) {  // warp-uniform: every lane holds the same cmax and vmax
                beta = vmax / cmax;
                vmax = cmax;
                rvmax = 1.f / cmax;
            }
            const float u0 = vq0 * rvmax, u1 = vq1 * rvmax;
            float alpha[2], mnew[2], p[4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                mnew[j] = fmaxf(mrun[j], mx[j]);
                const float a = (mnew[j] == -INFINITY) ? 1.f : exp2f(mrun[j] - mnew[j]);
                mrun[j] = mnew[j];
                lrun[j] *= a;
                alpha[j] = a * beta;
                const float e0 = (mnew[j] == -INFINITY) ? 0.f : exp2f(sacc[j] - mnew[j]);
                const float e1 = (mnew[j] == -INFINITY) ? 0.f : exp2f(sacc[2 + j] - mnew[j]);
                lrun[j] += e0 + e1;
                p[j] = e0 * u0;
                p[2 + j] = e1 * u1;
            }
            const uint32_t h01 = pack_f16(p[0], p[1]);
            const uint32_t h23 = pack_f16(p[2], p[3]);
            const float2 r01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
            const float2 r23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
            const uint32_t phi0 = movm_t(h01), phi1 = movm_t(h23);
            const uint32_t plo0 = movm_t(pack_f16(p[0] - r01.x, p[1] - r01.y));
            const uint32_t plo1 = movm_t(pack_f16(p[2] - r23.x, p[3] - r23.y));
            // ---- O^T = alpha * O^T + V^T P, two 16-d blocks per ldmatrix.x4.trans (rescale skipped
            // while no head's running max moved: alpha == 1 exactly)
            if (__any_sync(0xffffffffu, (alpha[0] != 1.f) | (alpha[1] != 1.f))) {
#pragma unroll
                for (int dt = 0; dt < D / 16; ++dt) {
                    o[dt][0] *= alpha[0];
                    o[dt][1] *= alpha[1];
                    o[dt][2] *= alpha[0];
                    o[dt][3] *= alpha[1];
                }
            }
#pragma unroll
            for (int dt = 0; dt < D / 16; dt += 2) {
                uint32_t r[4];
                ldsm_x4_t(vst + C::at(v_key, dt + v_seg), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    // r[2e]: keys 0-7, r[2e+1]: keys 8-15; bytes (k0,d) (k0,d+1) (k1,d) (k1,d+1)
                    const uint32_t lo = __byte_perm(r[2 * e], 0u, 0x3120);
                    const uint32_t hi = __byte_perm(r[2 * e + 1], 0u, 0x3120);
                    uint32_t a0, a1, a2, a3;  // a0 / a2: d even, a1 / a3: d odd
                    e4m3x4_to_f16x2x2(lo, a0, a1);
                    e4m3x4_to_f16x2x2(hi, a2, a3);
                    float(&od)[4] = o[dt + e];
                    mma_f16(od, a0, a1, a2, a3, phi0, phi1);
                    mma_f16(od, a0, a1, a2, a3, plo0, plo1);
                }
            }
            __syncwarp();  // stage s is free
        }
        cp_async_wait<0>();
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) lrun[j] += __shfl_xor_sync(0xffffffffu, lrun[j], off);
        }
        // O^T rows of block dt: row qn holds d = 16 dt + 2 qn, row qn + 8 holds d = 16 dt + 2 qn + 1
        if (SPLIT) {
            float* pb = part + static_cast<size_t>(it) * G * (D + 2);
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                const int d0 = dt * 16 + 2 * qn;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = hc + j;
                    if (h < G)
                        *reinterpret_cast<float2*>(pb + h * (D + 2) + d0) =
                            make_float2(o[dt][j] * vmax, o[dt][2 + j] * vmax);
                }
            }
            if (qn == 0) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = hc + j;
                    if (h < G) {
                        pb[h * (D + 2) + D] = mrun[j];
                        pb[h * (D + 2) + D + 1] = lrun[j];
                    }
                }
            }
            continue;
        }
        const float inv0 = lrun[0] > 0.f ? vmax / lrun[0] : 0.f;
        const float inv1 = lrun[1] > 0.f ? vmax / lrun[1] : 0.f;
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
            const int d0 = dt * 16 + 2 * qn;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = hc + j;
                if (h < G) {
                    const float inv = j ? inv1 : inv0;
                    const size_t ob = (static_cast<size_t>(b) * Hq + g * G + h) * D;
                    if (OUT_BF16) {
                        __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(O) + ob;
                        *reinterpret_cast<__nv_bfloat162*>(op + d0) =
                            __floats2bfloat162_rn(o[dt][j] * inv, o[dt][2 + j] * inv);
                    } else {
                        float* op = reinterpret_cast<float*>(O) + ob;
                        *reinterpret_cast<float2*>(op + d0) = make_float2(o[dt][j] * inv, o[dt][2 + j] * inv);
                    }
                }
            }
        }
    }
}

template <int D, int STAGES, int WARPS>
static cudaError_t launch_attn_fp8_t(const __nv_bfloat16* Q, const unsigned char* K8, const float* k_scale,
                                     const unsigned char* V8, const float* v_scale, const int* idx, int B, int Hq,
                                     int Hkv, int topk, float scale, void* O, bool out_bf16, KvPages pg, WsHeader* hdr,
                                     int num_sms, cudaStream_t stream) {
    using C = Fp8AttnCfg<D, STAGES, WARPS>;
    const long long units = static_cast<long long>(B) * Hkv;
    const int nchunks = (topk + C::CHUNK - 1) / C::CHUNK;
    int per = nchunks;
    const int splits = attn_splits(units, nchunks, WARPS, num_sms, &per);
    using KernFn = void (*)(const __nv_bfloat16*, const unsigned char*, const float*, const unsigned char*,
                            const float*, const int*, int, int, int, int, float, void*, int, int, float*, KvPages,
                            WsHeader*);
    static const KernFn table[2][2] = {
        {sparse_attn_fp8_kernel<D, STAGES, WARPS, false, false>, sparse_attn_fp8_kernel<D, STAGES, WARPS, false, true>},
        {sparse_attn_fp8_kernel<D, STAGES, WARPS, true, false>, sparse_attn_fp8_kernel<D, STAGES, WARPS, true, true>}};
    KernFn kern = table[out_bf16 ? 1 : 0][splits > 1 ? 1 : 0];
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
    if (e != cudaSuccess) return e;
    long long grid = num_sms;
    const long long need = (units * splits + WARPS - 1) / WARPS;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    float* part = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(hdr) + kWsHeaderBytes);
    kern<<<static_cast<int>(grid), WARPS * 32, C::SMEM, stream>>>(Q, K8, k_scale, V8, v_scale, idx, B, Hq, Hkv, topk,
                                                                   scale * 1.4426950408889634f, O, splits, per, part,
                                                                   pg, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess || splits == 1) return e;
    const int G = Hq / Hkv;
    if (splits > 32) return cudaErrorInvalidValue;
    if (out_bf16)
        attn_merge_kernel<D, true><<<static_cast<unsigned>(units), G * 32, 0, stream>>>(part, G, splits, Hq, Hkv, O);
    else
        attn_merge_kernel<D, false><<<static_cast<unsigned>(units), G * 32, 0, stream>>>(part, G, splits, Hq, Hkv, O);
    return cudaGetLastError();
}

// Bytes of split-range state the sparse attention needs beyond the status word: the larger of
// the bf16 kernel's and (one query per sequence) the fp8 kernel's ranges for this shape.
size_t sparse_attn_part_bytes(int B, int n_q, int Hq, int Hkv, int d, int topk, int num_sms) {
    if (d != 128 && d != 64) return 0;
    const long long units = static_cast<long long>(B) * n_q * Hkv;
    int per = 0;
    const bool dec = attn_decode_shape(units, d, num_sms);
    const int chunk = dec ? kAttnDecodeChunkD128 : 16;
    const int warps = dec ? kAttnDecodeWarpsD128 : d == 128 ? kAttnWarpsD128 : kAttnWarpsD64;
    int splits = attn_splits(units, (topk + chunk - 1) / chunk, warps, num_sms, &per);
    if (n_q == 1) {
        const int s8 = attn_splits(units, (topk + 15) / 16, d == 128 ? kAttnFp8WarpsD128 : kAttnFp8WarpsD64, num_sms,
                                   &per);
        if (s8 > splits) splits = s8;
    }
    if (splits == 1) return 0;
    return static_cast<size_t>(units) * splits * (Hq / Hkv) * (d + 2) * sizeof(float);
}

// Host dispatcher: returns cudaErrorNotSupported for shapes without a kernel.
cudaError_t launch_sparse_attn(const void* Q, const void* K, const void* V, const int* idx, int B, int n_q,
                               int n_kv, int Hq, int Hkv, int d, int topk, float scale, void* O, bool out_bf16,
                               IdxShare share, KvPages pg, WsHeader* hdr, int num_sms, cudaStream_t stream) {
    auto q = static_cast<const __nv_bfloat16*>(Q);
    auto k = static_cast<const __nv_bfloat16*>(K);
    auto v = static_cast<const __nv_bfloat16*>(V);
    // 16-key chunks, 2 stages per warp, swizzled rows: as many warps per SM as shared memory
    // holds (measured on B200: warps in flight matter more than stages per warp); 32-key
    // chunks for decode shapes at d = 128.
    const long long units = static_cast<long long>(B) * n_q * Hkv;
    if (d == 128 && attn_decode_shape(units, d, num_sms))
        return launch_attn_t<128, kAttnDecodeChunkD128, 2, kAttnDecodeWarpsD128, true, true>(
            q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, share, pg, hdr, num_sms, stream);
    if (d == 128)
        return launch_attn_t<128, 16, 2, kAttnWarpsD128, true, true>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O,
                                                         out_bf16, share, pg, hdr, num_sms, stream);
    if (d == 64)
        return launch_attn_t<64, 16, 2, kAttnWarpsD64, true, true>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O,
                                                        out_bf16, share, pg, hdr, num_sms, stream);
    return cudaErrorNotSupported;
}

// fp8 (E4M3 + per-row scale) paged K/V: one query per sequence.
cudaError_t launch_sparse_attn_fp8_paged(const void* Q, const void* K8, const float* k_scale, const void* V8,
                                         const float* v_scale, const int* idx, int B, int Hq, int Hkv, int d, int topk,
                                         float scale, void* O, bool out_bf16, KvPages pg, WsHeader* hdr, int num_sms,
                                         cudaStream_t stream) {
    auto q = static_cast<const __nv_bfloat16*>(Q);
    auto k = static_cast<const unsigned char*>(K8);
    auto v = static_cast<const unsigned char*>(V8);
    if (d == 128)
        return launch_attn_fp8_t<128, kAttnFp8StagesD128, kAttnFp8WarpsD128>(
            q, k, k_scale, v, v_scale, idx, B, Hq, Hkv, topk, scale, O, out_bf16, pg, hdr, num_sms, stream);
    if (d == 64)
        return launch_attn_fp8_t<64, kAttnFp8StagesD64, kAttnFp8WarpsD64>(q, k, k_scale, v, v_scale, idx, B, Hq, Hkv,
                                                                         topk, scale, O, out_bf16, pg, hdr, num_sms,
                                                                         stream);
    return cudaErrorNotSupported;
}

}  // namespace dsa
