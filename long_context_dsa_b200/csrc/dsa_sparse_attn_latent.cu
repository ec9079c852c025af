// dsa_sparse_attn_latent.cu -- sparse attention over a shared latent row per
// token (MLA-style): the row's 576 dims are the key of every query head and
// its first 512 dims the value.
//
// [Explainer] §稀疏注意力的隐性开销: each token attends only to its top-k
// history tokens.  The latent layout itself is this library's reading for
// the 1M-token configuration (the pages do not describe the KV layout).
//
// Design: one CTA per (query row, block of 8*WARPS query heads).  All warps
// share the gathered rows: the CTA streams the selected tokens' latent rows
// (1152 bytes each) through a cp.async ring, 16 tokens per stage, and every
// warp computes its 8 heads on each stage with warp-level bf16 MMAs:
// S^T = K Q^T (keys on M, the warp's 8 heads on N, K = 576) and
// O^T += V^T P (d on M: 32 tiles of 16 for d_v = 512, kept in registers).
// The query block is staged in shared memory once per row.  P moves into the
// B-operand layout with movmatrix and is split into bf16 hi + lo parts.
#include "dsa_common.cuh"

namespace dsa {

namespace lat {

constexpr int DQK = 576, DV = 512;
constexpr int CHUNK = 16;                 // tokens per stage
constexpr int STAGES = 4;
constexpr int RS = DQK * 2 + 16;          // padded row stride (bank-conflict-free ldmatrix)
constexpr int SEGS = DQK * 2 / 16;        // 72 16-byte segments per row

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
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int WARPS>
struct Cfg {
    static constexpr int HB = 8 * WARPS;  // query heads per CTA
    static constexpr int Q_BYTES = HB * RS;
    static constexpr int STAGE_BYTES = CHUNK * RS;
    static constexpr size_t SMEM = Q_BYTES + static_cast<size_t>(STAGES) * STAGE_BYTES + STAGES * CHUNK * 4;
};

// SPLIT: each (query row, head block) unit is cut into `splits` ranges of `cps` chunks (few
// rows, e.g. one decode token: the ranges spread over the SMs); a range writes its unnormalised
// O and its (max, sum) per head to `part` and latent_merge_kernel combines the ranges.
template <int WARPS, bool OUT_BF16, bool SPLIT>
__global__ void __launch_bounds__(WARPS * 32, 1)
    latent_attn_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ KV,
                       const int* __restrict__ idx, int B, int n_q, int n_kv, int Hq, int topk, float scale_log2,
                       void* __restrict__ O, int splits, int cps, float* __restrict__ part, IdxShare share,
                       WsHeader* hdr) {
    using C = Cfg<WARPS>;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* sq = smem;
    unsigned char* ring = smem + C::Q_BYTES;
    int* sidx = reinterpret_cast<int*>(ring + STAGES * C::STAGE_BYTES);
    const uint32_t sq_s = smem_u32(sq), ring_s = smem_u32(ring);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthr = WARPS * 32;
    const int hblocks = Hq / C::HB;
    const long long units = static_cast<long long>(B) * n_q * hblocks;
    const long long items = SPLIT ? units * splits : units;
    const int nchunks = (topk + CHUNK - 1) / CHUNK;

    const int qn = lane >> 2, hc = 2 * (lane & 3);
    const int lrow = lane & 7, lq = lane >> 3;
    const int k_key_off = ((lq & 1) ? 8 : 0) + lrow, k_d_off = (lq >= 2) ? 8 : 0;   // K: non-trans A
    const int v_key_off = ((lq >= 2) ? 8 : 0) + lrow, v_d_off = (lq & 1) ? 8 : 0;  // V: trans A
    // Q^T B fragments via ldmatrix.x4 over two k-steps: rows = heads, 8-element column groups
    const int q_row = lane & 7, q_col = (lane >> 3) * 8;

    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const long long u = SPLIT ? it / splits : it;
        const int sp = SPLIT ? static_cast<int>(it % splits) : 0;
        const int c0 = SPLIT ? sp * cps : 0;                       // this item's chunk range
        const int c1 = SPLIT ? min(nchunks, c0 + cps) : nchunks;
        const long long row = u / hblocks;
        const int hb = static_cast<int>(u % hblocks);
        const long long b = row / n_q;
        const int qi = static_cast<int>(row - b * n_q);
        const int* irow = idx + (b * share.rows(n_q) + qi / share.q_per_idx) * topk;
        const int lim = share.limit(qi);  // shared rows: keys past this query's own position are skipped
        const __nv_bfloat16* kvb = KV + static_cast<size_t>(b) * n_kv * DQK;

        __syncthreads();  // the previous unit is done with the query block and the ring
        // query block -> shared (its own cp.async group, retired with the first stage)
        {
            const __nv_bfloat16* qb = Q + (static_cast<size_t>(row) * Hq + hb * C::HB) * DQK;
            for (int sgi = threadIdx.x; sgi < C::HB * SEGS; sgi += nthr) {
                const int h = sgi / SEGS, sg = sgi % SEGS;
                cp_async16(sq_s + h * RS + sg * 16, qb + static_cast<size_t>(h) * DQK + sg * 8, 16u);
            }
        }
        auto issue = [&](int c) {
            if (c < c1) {
                const int s = (c - c0) % STAGES;
                if (threadIdx.x < CHUNK) {
                    const int kk = c * CHUNK + threadIdx.x;
                    int t = kk < topk ? __ldg(irow + kk) : -1;
                    if (t < -1 || t >= n_kv) {
                        raise_status(hdr, DSA_STATUS_BAD_INDEX, t);
                        t = -1;
                    }
                    sidx[s * CHUNK + threadIdx.x] = t > lim ? -1 : t;
                }
                for (int sgi = threadIdx.x; sgi < CHUNK * SEGS; sgi += nthr) {
                    const int key = sgi / SEGS, sg = sgi % SEGS;
                    const int kk = c * CHUNK + key;
                    int t = kk < topk ? __ldg(irow + kk) : -1;
                    const bool ok = t >= 0 && t < n_kv && t <= lim;
                    cp_async16(ring_s + s * C::STAGE_BYTES + key * RS + sg * 16,
                               kvb + static_cast<size_t>(ok ? t : 0) * DQK + sg * 8, ok ? 16u : 0u);
                }
            }
            cp_async_commit();
        };

        float o[DV / 16][4];
#pragma unroll
        for (int i = 0; i < DV / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};
        const uint32_t qw = sq_s + (warp * 8 + q_row) * RS + q_col * 2;  // this lane's ldmatrix row of Q

#pragma unroll
        for (int c = c0; c < c0 + STAGES - 1; ++c) issue(c);
        for (int c = c0; c < c1; ++c) {
            issue(c + STAGES - 1);
            cp_async_wait<STAGES - 1>();
            __syncthreads();
            const int s = (c - c0) % STAGES;
            const uint32_t kst = ring_s + s * C::STAGE_BYTES;
            const int* si = sidx + s * CHUNK;
            // ---- S^T = K Q^T over 36 k-steps (two per ldmatrix.x4 of Q)
            float sacc[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t abase = kst + k_key_off * RS + k_d_off * 2;
#pragma unroll 6
            for (int kp = 0; kp < DQK / 32; ++kp) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(qw + kp * 64, b0, b1, b2, b3);
                uint32_t a0, a1, a2, a3;
                ldsm_x4(abase + kp * 64, a0, a1, a2, a3);
                mma_bf16(sacc, a0, a1, a2, a3, b0, b1);
                ldsm_x4(abase + kp * 64 + 32, a0, a1, a2, a3);
                mma_bf16(s2, a0, a1, a2, a3, b2, b3);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[e] += s2[e];
            // ---- mask, scale, online softmax
            const bool v0 = si[qn] >= 0, v1 = si[qn + 8] >= 0;
            float mx[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                sacc[j] = v0 ? sacc[j] * scale_log2 : -INFINITY;
                sacc[2 + j] = v1 ? sacc[2 + j] * scale_log2 : -INFINITY;
                mx[j] = fmaxf(sacc[j], sacc[2 + j]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], off));
            }
            float alpha[2], mnew[2], p[4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                mnew[j] = fmaxf(mrun[j], mx[j]);
                alpha[j] = (mnew[j] == -INFINITY) ? 1.f : exp2f(mrun[j] - mnew[j]);
                mrun[j] = mnew[j];
                p[j] = (mnew[j] == -INFINITY) ? 0.f : exp2f(sacc[j] - mnew[j]);
                p[2 + j] = (mnew[j] == -INFINITY) ? 0.f : exp2f(sacc[2 + j] - mnew[j]);
                lrun[j] = lrun[j] * alpha[j] + p[j] + p[2 + j];
            }
            const uint32_t h01 = pack_bf16(p[0], p[1]), h23 = pack_bf16(p[2], p[3]);
            const __nv_bfloat162 hh01 = *reinterpret_cast<const __nv_bfloat162*>(&h01);
            const __nv_bfloat162 hh23 = *reinterpret_cast<const __nv_bfloat162*>(&h23);
            const uint32_t phi0 = movm_t(h01), phi1 = movm_t(h23);
            const uint32_t plo0 = movm_t(pack_bf16(p[0] - __low2float(hh01), p[1] - __high2float(hh01)));
            const uint32_t plo1 = movm_t(pack_bf16(p[2] - __low2float(hh23), p[3] - __high2float(hh23)));
            // ---- O^T = alpha * O^T + V^T P  (V = first 512 dims of the latent rows)
            const uint32_t vbase = kst + v_key_off * RS + v_d_off * 2;
#pragma unroll
            for (int dt = 0; dt < DV / 16; ++dt) {
                o[dt][0] *= alpha[0];
                o[dt][1] *= alpha[1];
                o[dt][2] *= alpha[0];
                o[dt][3] *= alpha[1];
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(vbase + dt * 32, a0, a1, a2, a3);
                mma_bf16(o[dt], a0, a1, a2, a3, phi0, phi1);
                mma_bf16(o[dt], a0, a1, a2, a3, plo0, plo1);
            }
            __syncthreads();  // stage s may be refilled
        }
        cp_async_wait<0>();
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) lrun[j] += __shfl_xor_sync(0xffffffffu, lrun[j], off);
        }
        if (SPLIT) {
            // unnormalised O^T and (max, sum) of this range, per head: [item][head][DV + 2]
#pragma unroll
            for (int dt = 0; dt < DV / 16; ++dt) {
                const int d0 = dt * 16 + qn;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float* pp = part + (static_cast<size_t>(it) * C::HB + warp * 8 + hc + j) * (DV + 2);
                    pp[d0] = o[dt][j];
                    pp[d0 + 8] = o[dt][2 + j];
                }
            }
            if (qn == 0) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float* pp = part + (static_cast<size_t>(it) * C::HB + warp * 8 + hc + j) * (DV + 2);
                    pp[DV] = mrun[j];
                    pp[DV + 1] = lrun[j];
                }
            }
            continue;
        }
        const float inv0 = lrun[0] > 0.f ? 1.f / lrun[0] : 0.f;
        const float inv1 = lrun[1] > 0.f ? 1.f / lrun[1] : 0.f;
#pragma unroll
        for (int dt = 0; dt < DV / 16; ++dt) {
            const int d0 = dt * 16 + qn;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = hb * C::HB + warp * 8 + hc + j;
                const float inv = j ? inv1 : inv0;
                const size_t ob = (static_cast<size_t>(row) * Hq + h) * DV;
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

// Combine the split ranges of each (query row, head block): for every head,
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s with M = max_s m_s (a range that met only
// skipped entries has m_s = -inf and drops out).  One 128-thread block per (unit, head, 128
// output columns): every thread issues the loads of its column in all ranges (splits <= 32) at
// once, the first warp meanwhile turns the ranges' (m, l) into weights in shared memory, and the
// thread then sums its column.  Four blocks per head spread one query row's merge over the SMs.
template <bool OUT_BF16>
__global__ void __launch_bounds__(128)
    latent_merge_kernel(const float* __restrict__ part, int HB, int hblocks, int splits, int Hq,
                        void* __restrict__ O) {
    constexpr int CB = DV / 128;  // column blocks per head
    __shared__ float wt[32];
    __shared__ float inv_l;
    const long long uh = blockIdx.x / CB;  // (unit, head)
    const int cb = static_cast<int>(blockIdx.x % CB);
    const long long u = uh / HB;           // (row, head block)
    const int h = static_cast<int>(uh % HB);
    const long long row = u / hblocks;
    const int hb = static_cast<int>(u % hblocks);
    const size_t sstride = static_cast<size_t>(HB) * (DV + 2);
    const float* p0 = part + (static_cast<size_t>(u) * splits * HB + h) * (DV + 2);
    const int d = cb * 128 + threadIdx.x;
    float v[32];
#pragma unroll
    for (int s2 = 0; s2 < 32; ++s2) v[s2] = s2 < splits ? __ldg(p0 + s2 * sstride + d) : 0.f;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const float m = lane < splits ? __ldg(p0 + lane * sstride + DV) : -INFINITY;
        const float l = lane < splits ? __ldg(p0 + lane * sstride + DV + 1) : 0.f;
        float M = m;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
        float L = f * l;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        wt[lane] = f;
        if (lane == 0) inv_l = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
    float acc = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 32; ++s2)
        if (s2 < splits) acc = fmaf(wt[s2], v[s2], acc);
    const float out = acc * inv_l;
    const size_t ob = (static_cast<size_t>(row) * Hq + static_cast<size_t>(hb) * HB + h) * DV + d;
    if (OUT_BF16)
        reinterpret_cast<__nv_bfloat16*>(O)[ob] = __float2bfloat16_rn(out);
    else
        reinterpret_cast<float*>(O)[ob] = out;
}

}  // namespace lat

cudaError_t launch_latent_merge(const float* part, int HB, int hblocks, int splits, long long units, int Hq, void* O,
                                bool out_bf16, cudaStream_t stream) {
    if (splits > 32) return cudaErrorInvalidValue;  // one lane per range in the merge
    const unsigned mblocks = static_cast<unsigned>(units * HB * (lat::DV / 128));
    if (out_bf16)
        lat::latent_merge_kernel<true><<<mblocks, 128, 0, stream>>>(part, HB, hblocks, splits, Hq, O);
    else
        lat::latent_merge_kernel<false><<<mblocks, 128, 0, stream>>>(part, HB, hblocks, splits, Hq, O);
    return cudaGetLastError();
}

namespace lat {

// Warps per CTA (8 query heads each) for Hq query heads.
inline int warps_for(int Hq) { return Hq % 64 == 0 ? 8 : Hq % 32 == 0 ? 4 : Hq % 16 == 0 ? 2 : 1; }

// Ranges per (row, head block) unit: 1 when the units alone fill every SM; otherwise enough to
// give each SM about one item, at most 32 ranges and at least 2 chunks (32 keys) each.  Depends
// only on the shape and the SM count, so the workspace query and the launch agree.
inline int latent_splits(long long units, int nchunks, int num_sms, int* cps) {
    int s = 1;
    if (units < num_sms) {
        s = static_cast<int>((num_sms + units - 1) / units);
        const int most = nchunks / 2 > 1 ? nchunks / 2 : 1;
        if (s > most) s = most;
        if (s > 32) s = 32;
    }
    *cps = (nchunks + s - 1) / s;
    return (nchunks + *cps - 1) / *cps;
}

template <int WARPS>
cudaError_t launch_w(const void* Q, const void* KV, const int* idx, int B, int n_q, int n_kv, int Hq, int topk,
                     float scale, void* O, bool out_bf16, IdxShare share, WsHeader* hdr, int num_sms,
                     cudaStream_t stream) {
    using Cf = Cfg<WARPS>;
    const int hblocks = Hq / Cf::HB;
    const long long units = static_cast<long long>(B) * n_q * hblocks;
    const int nchunks = (topk + CHUNK - 1) / CHUNK;
    int cps = nchunks;
    const int splits = latent_splits(units, nchunks, num_sms, &cps);
    auto kern = out_bf16 ? (splits > 1 ? latent_attn_kernel<WARPS, true, true> : latent_attn_kernel<WARPS, true, false>)
                         : (splits > 1 ? latent_attn_kernel<WARPS, false, true> : latent_attn_kernel<WARPS, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Cf::SMEM));
    if (e != cudaSuccess) return e;
    const long long items = units * splits;
    long long grid = num_sms;
    if (grid > items) grid = items;
    if (grid < 1) grid = 1;
    float* part = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(hdr) + kWsHeaderBytes);
    kern<<<static_cast<int>(grid), WARPS * 32, Cf::SMEM, stream>>>(
        static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(KV), idx, B, n_q, n_kv, Hq, topk,
        scale * 1.4426950408889634f, O, splits, cps, part, share, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess || splits == 1) return e;
    return launch_latent_merge(part, Cf::HB, hblocks, splits, units, Hq, O, out_bf16, stream);
}

}  // namespace lat

bool latent_tc_applies(int Hq);
cudaError_t launch_latent_tc(const void* Q, const void* KV, const int* idx, int B, int n_q, int n_kv, int Hq,
                             int topk, float scale, void* O, bool out_bf16, IdxShare share, WsHeader* hdr,
                             int max_splits, int num_sms, cudaStream_t stream);

// Many query rows with heads in blocks of 64: the tensor-core kernel (dsa_latent_tc.cu).  Otherwise
// (decode, a few rows, other head counts) the warp-MMA kernel above, with split ranges when the
// rows alone cannot fill the GPU.
cudaError_t launch_sparse_attn_latent(const void* Q, const void* KV, const int* idx, int B, int n_q, int n_kv,
                                      int Hq, int topk, float scale, void* O, bool out_bf16, IdxShare share,
                                      WsHeader* hdr, int num_sms, cudaStream_t stream) {
    if (latent_tc_applies(Hq)) {
        const long long units = static_cast<long long>(B) * n_q * (Hq / 64);
        int cps = 0;
        const int max_splits = lat::latent_splits(units, (topk + lat::CHUNK - 1) / lat::CHUNK, num_sms, &cps);
        return launch_latent_tc(Q, KV, idx, B, n_q, n_kv, Hq, topk, scale, O, out_bf16, share, hdr, max_splits,
                                num_sms, stream);
    }
    switch (lat::warps_for(Hq)) {
        case 8: return lat::launch_w<8>(Q, KV, idx, B, n_q, n_kv, Hq, topk, scale, O, out_bf16, share, hdr, num_sms, stream);
        case 4: return lat::launch_w<4>(Q, KV, idx, B, n_q, n_kv, Hq, topk, scale, O, out_bf16, share, hdr, num_sms, stream);
        case 2: return lat::launch_w<2>(Q, KV, idx, B, n_q, n_kv, Hq, topk, scale, O, out_bf16, share, hdr, num_sms, stream);
        default:
            if (Hq % 8 != 0) return cudaErrorNotSupported;
            return lat::launch_w<1>(Q, KV, idx, B, n_q, n_kv, Hq, topk, scale, O, out_bf16, share, hdr, num_sms, stream);
    }
}

// Bytes of split-range state the latent attention needs beyond the status word.
size_t sparse_attn_latent_part_bytes(int B, int n_q, int Hq, int topk, int num_sms) {
    if (Hq < 8 || Hq % 8 != 0) return 0;
    const int HB = 8 * lat::warps_for(Hq);
    const long long units = static_cast<long long>(B) * n_q * (Hq / HB);
    int cps = 0;
    const int splits = lat::latent_splits(units, (topk + lat::CHUNK - 1) / lat::CHUNK, num_sms, &cps);
    if (splits == 1) return 0;
    return static_cast<size_t>(units) * splits * HB * (lat::DV + 2) * sizeof(float);
}

}  // namespace dsa
