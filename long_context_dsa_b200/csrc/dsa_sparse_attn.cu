// dsa_sparse_attn.cu -- attention over each query's selected tokens (K3).
//
// [Explainer] §稀疏注意力的隐性开销: every token attends only to its top-k
// history tokens; §IndexShare 的共享机制: S layers keep their own attention
// weights, so each layer runs this kernel with its own Q/K/V.
//
// Design (B200): the work is a gather -- every query reads k rows of K and
// V picked by the index cache -- so it is bound by HBM, not by math.
//   * A persistent CTA owns (query row, block of HB KV heads) items.  One
//     producer warp streams the selected rows into a multi-stage shared
//     memory ring with one bulk async copy (cp.async.bulk, TMA engine) per
//     gathered row: a row of HB*D bf16 is contiguous in the token-major
//     K/V layout.  Completion is tracked by mbarrier transaction bytes.
//   * HB consumer warps, one per KV head, run an online-softmax attention
//     over the chunk with warp-level bf16 tensor-core MMAs (m16n8k16):
//     S^T = K_chunk Q^T puts keys on M and the GQA group's query heads on
//     N (8 columns, no padding at G = 8); O^T += V^T P uses d on M.  The
//     probabilities move from the S^T accumulator layout into the B
//     operand layout with movmatrix.  P is split into bf16 hi + lo parts
//     (two MMAs) so the weights keep ~16 bits of precision.
//   * Rows are stored at a stride of RB+16 bytes, which makes every
//     ldmatrix conflict-free without swizzling the copies.
#include "dsa_common.cuh"

namespace dsa {

static constexpr int kAttnChunk = 32;  // gathered keys per pipeline stage

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

template <int D, int HB, int STAGES>
struct AttnCfg {
    static constexpr int RB = HB * D * 2;         // bytes of one gathered row (HB heads)
    static constexpr int RS = RB + 16;            // smem row stride (bank-conflict free)
    static constexpr int STAGE_BYTES = 2 * kAttnChunk * RS;
    static constexpr int THREADS = (HB + 1) * 32;
    static constexpr size_t SMEM = static_cast<size_t>(STAGES) * STAGE_BYTES + STAGES * kAttnChunk * 4 +
                                   2 * STAGES * 8 + 16;
};

template <int D, int HB, int STAGES, bool OUT_BF16>
__global__ void __launch_bounds__(AttnCfg<D, HB, STAGES>::THREADS, 1)
    sparse_attn_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                       const __nv_bfloat16* __restrict__ V, const int* __restrict__ idx, int B, int n_q,
                       int n_kv, int Hq, int Hkv, int topk, float scale_log2, void* __restrict__ O,
                       WsHeader* hdr) {
    using C = AttnCfg<D, HB, STAGES>;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* stage_base = smem;
    int* sidx = reinterpret_cast<int*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(sidx + STAGES * kAttnChunk);
    uint64_t* empty = full + STAGES;
    int* abort_flag = reinterpret_cast<int*>(empty + STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = Hq / Hkv;
    const int hblocks = Hkv / HB;
    const long long total = static_cast<long long>(B) * n_q * hblocks;
    const int nchunks = (topk + kAttnChunk - 1) / kAttnChunk;

    // zero the ring once: rows never written by a copy must hold finite data
    for (int i = threadIdx.x; i < STAGES * C::STAGE_BYTES / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(stage_base)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], HB);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    fence_proxy_async_smem();
    __syncthreads();

    if (warp == HB) {
        // ------------------------------------------------------------ producer
        int last_round[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
        long long it = 0;
        bool ok_run = true;
        for (long long w = blockIdx.x; w < total && ok_run; w += gridDim.x) {
            const long long row = w / hblocks;
            const int hb = static_cast<int>(w % hblocks);
            const long long b = row / n_q;
            const int* irow = idx + row * topk;
            const size_t tok_stride = static_cast<size_t>(Hkv) * D;  // elements per token
            const __nv_bfloat16* kb = K + static_cast<size_t>(b) * n_kv * tok_stride + static_cast<size_t>(hb) * HB * D;
            const __nv_bfloat16* vb = V + static_cast<size_t>(b) * n_kv * tok_stride + static_cast<size_t>(hb) * HB * D;
            for (int c = 0; c < nchunks; ++c, ++it) {
                const int s = static_cast<int>(it % STAGES);
                const int r = static_cast<int>(it / STAGES);
                if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1)) {
                    if (lane == 0) raise_status(hdr, DSA_STATUS_TIMEOUT, 0x5a01);
                    ok_run = false;
                    break;
                }
                const int kk = c * kAttnChunk + lane;
                const int t = (kk < topk) ? __ldg(irow + kk) : -1;
                const bool ok = (t >= 0) && (t < n_kv);
                if (t < -1 || t >= n_kv) raise_status(hdr, DSA_STATUS_BAD_INDEX, t);
                sidx[s * kAttnChunk + lane] = ok ? t : -1;
                const unsigned m = __ballot_sync(0xffffffffu, ok);
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(__popc(m)) * 2u * C::RB);
                __syncwarp();
                if (ok) {
                    unsigned char* krow = stage_base + s * C::STAGE_BYTES + lane * C::RS;
                    unsigned char* vrow = krow + kAttnChunk * C::RS;
                    bulk_g2s(krow, kb + static_cast<size_t>(t) * tok_stride, C::RB, &full[s]);
                    bulk_g2s(vrow, vb + static_cast<size_t>(t) * tok_stride, C::RB, &full[s]);
                }
                last_round[s] = r;
            }
            if (__any_sync(0xffffffffu, *reinterpret_cast<volatile int*>(abort_flag) != 0)) break;
        }
        if (!ok_run && lane == 0) atomicExch(abort_flag, 1);
        // never leave with copies in flight into this CTA's shared memory
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            if (last_round[s] >= 0 && !mbar_wait(&full[s], last_round[s] & 1) && lane == 0)
                raise_status(hdr, DSA_STATUS_TIMEOUT, 0x5a02);
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int cw = warp;  // KV head within the block
    const int qn = lane >> 2;          // query head (N column) this lane loads for Q
    const int hc = 2 * (lane & 3);     // first of the two head columns this lane owns in C tiles
    const int lrow = lane & 7, lq = lane >> 3;
    // ldmatrix lane offsets
    const int k_key_off = ((lq & 1) ? 8 : 0) + lrow, k_d_off = (lq >= 2) ? 8 : 0;   // K: non-trans A
    const int v_key_off = ((lq >= 2) ? 8 : 0) + lrow, v_d_off = (lq & 1) ? 8 : 0;  // V: trans A
    long long it = 0;
    for (long long w = blockIdx.x; w < total; w += gridDim.x) {
        const long long row = w / hblocks;
        const int hb = static_cast<int>(w % hblocks);
        const int g = hb * HB + cw;  // KV head
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
        float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};

        bool alive = true;
        for (int c = 0; c < nchunks; ++c, ++it) {
            const int s = static_cast<int>(it % STAGES);
            const int r = static_cast<int>(it / STAGES);
            if (!mbar_wait(&full[s], r & 1)) {
                if (lane == 0) {
                    raise_status(hdr, DSA_STATUS_TIMEOUT, 0x5a03);
                    atomicExch(abort_flag, 1);
                }
                alive = false;
                break;
            }
            const unsigned char* kst = stage_base + s * C::STAGE_BYTES;
            const unsigned char* vst = kst + kAttnChunk * C::RS;
            const int* si = sidx + s * kAttnChunk;
            // ---- S^T = K Q^T  (two 16-key tiles)
            float sacc[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                sacc[mt][0] = sacc[mt][1] = sacc[mt][2] = sacc[mt][3] = 0.f;
                const uint32_t abase =
                    smem_u32(kst + (mt * 16 + k_key_off) * C::RS + (cw * D + k_d_off) * 2);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(abase + ks * 32, a0, a1, a2, a3);
                    mma_bf16(sacc[mt], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                }
            }
            // ---- mask, scale, online softmax
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
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
                alpha[j] = (mnew[j] == -INFINITY) ? 1.f : exp2f(mrun[j] - mnew[j]);
                mrun[j] = mnew[j];
                lrun[j] *= alpha[j];
            }
            uint32_t phi[2][2], plo[2][2];  // [k-step][matrix rows 0-7 / 8-15]
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                float p[4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    p[j] = (mnew[j] == -INFINITY) ? 0.f : exp2f(sacc[mt][j] - mnew[j]);
                    p[2 + j] = (mnew[j] == -INFINITY) ? 0.f : exp2f(sacc[mt][2 + j] - mnew[j]);
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
            // ---- O^T = alpha * O^T + V^T P
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                o[dt][0] *= alpha[0];
                o[dt][1] *= alpha[1];
                o[dt][2] *= alpha[0];
                o[dt][3] *= alpha[1];
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(smem_u32(vst + (ks * 16 + v_key_off) * C::RS + (cw * D + dt * 16 + v_d_off) * 2), a0,
                              a1, a2, a3);
                    mma_bf16(o[dt], a0, a1, a2, a3, phi[ks][0], phi[ks][1]);
                    mma_bf16(o[dt], a0, a1, a2, a3, plo[ks][0], plo[ks][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (!alive) break;
        // ---- finalize: row sums across the 8 lanes sharing a head column
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) lrun[j] += __shfl_xor_sync(0xffffffffu, lrun[j], off);
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
        if (*reinterpret_cast<volatile int*>(abort_flag) != 0) break;
    }
}

template <int D, int HB, int STAGES>
static cudaError_t launch_attn_t(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                                 const int* idx, int B, int n_q, int n_kv, int Hq, int Hkv, int topk,
                                 float scale, void* O, bool out_bf16, WsHeader* hdr, int num_sms,
                                 cudaStream_t stream) {
    using C = AttnCfg<D, HB, STAGES>;
    auto kern = out_bf16 ? sparse_attn_kernel<D, HB, STAGES, true> : sparse_attn_kernel<D, HB, STAGES, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
    if (e != cudaSuccess) return e;
    const long long total = static_cast<long long>(B) * n_q * (Hkv / HB);
    long long grid = num_sms;
    if (grid > total) grid = total;
    if (grid < 1) grid = 1;
    const float scale_log2 = scale * 1.4426950408889634f;
    kern<<<static_cast<int>(grid), C::THREADS, C::SMEM, stream>>>(Q, K, V, idx, B, n_q, n_kv, Hq, Hkv, topk,
                                                                  scale_log2, O, hdr);
    return cudaGetLastError();
}

// Host dispatcher: returns cudaErrorNotSupported for shapes without a kernel.
cudaError_t launch_sparse_attn(const void* Q, const void* K, const void* V, const int* idx, int B, int n_q,
                               int n_kv, int Hq, int Hkv, int d, int topk, float scale, void* O, bool out_bf16,
                               WsHeader* hdr, int num_sms, cudaStream_t stream) {
    auto q = static_cast<const __nv_bfloat16*>(Q);
    auto k = static_cast<const __nv_bfloat16*>(K);
    auto v = static_cast<const __nv_bfloat16*>(V);
    if (d == 128) {
        if (Hkv % 4 == 0)
            return launch_attn_t<128, 4, 3>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, hdr, num_sms, stream);
        if (Hkv % 2 == 0)
            return launch_attn_t<128, 2, 4>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, hdr, num_sms, stream);
        return launch_attn_t<128, 1, 6>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, hdr, num_sms, stream);
    }
    if (d == 64) {
        if (Hkv % 8 == 0)
            return launch_attn_t<64, 8, 3>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, hdr, num_sms, stream);
        if (Hkv % 4 == 0)
            return launch_attn_t<64, 4, 4>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, hdr, num_sms, stream);
        return launch_attn_t<64, 1, 6>(q, k, v, idx, B, n_q, n_kv, Hq, Hkv, topk, scale, O, out_bf16, hdr, num_sms, stream);
    }
    return cudaErrorNotSupported;
}

}  // namespace dsa
