// dsa_pattern.cu -- choosing which layers of a group run the indexer (F) and
// which reuse the most recent F layer's selection (S).
//
// [QbitAI] §IndexCache: for an existing model the layers worth keeping are
// searched by how the loss changes; [Explainer] §训练无关: a greedy pass over a
// small calibration batch decides the F and S layers without touching the
// weights.  Without trained weights the loss here is a proxy the pages also
// report (adjacent layers pick 70-100% of the same tokens): an S layer that
// reuses F layer f's selection loses the part of its own top-k that f's
// top-k misses.
//
//   * overlap_count_kernel: |A_r ∩ B_r| per row of two index buffers in the
//     canonical layout (ascending indices, then -1), one warp per row: each
//     lane binary-searches its entries of A in B.
//   * layer_pattern_search (host): greedy removal from the all-F pattern.
#include <cstring>

#include "dsa_common.cuh"

namespace dsa {

__global__ void overlap_count_kernel(const int* __restrict__ a, const int* __restrict__ b, long long rows, int k,
                                     int* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long r = w0; r < rows; r += nw) {
        const int* ra = a + r * k;
        const int* rb = b + r * k;
        // valid entries of B: the first -1 ends them
        int lo = 0, hi = k;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(rb + mid) < 0)
                hi = mid;
            else
                lo = mid + 1;
        }
        const int nb = lo;
        int c = 0;
        for (int i = lane; i < k; i += 32) {
            const int x = __ldg(ra + i);
            if (x < 0) continue;
            int l2 = 0, h2 = nb;
            while (l2 < h2) {
                const int mid = (l2 + h2) >> 1;
                if (__ldg(rb + mid) < x)
                    l2 = mid + 1;
                else
                    h2 = mid;
            }
            c += (l2 < nb && __ldg(rb + l2) == x) ? 1 : 0;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
        if (lane == 0) out[r] = c;
    }
}

cudaError_t launch_overlap_count(const int* a, const int* b, long long rows, int k, int* out, int num_sms,
                                 cudaStream_t stream) {
    long long blocks = (rows + 7) / 8;  // 8 warps a block
    const long long cap = 8ll * num_sms;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    overlap_count_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(a, b, rows, k, out);
    return cudaGetLastError();
}

// Proxy loss of a pattern: sum over S layers j of (1 - overlap[f][j]), f the most
// recent F layer before j.
static double pattern_loss(const double* ov, int n, const char* pat) {
    double loss = 0.0;
    int f = 0;
    for (int j = 0; j < n; ++j) {
        if (pat[j] == 'F')
            f = j;
        else
            loss += 1.0 - ov[static_cast<size_t>(f) * n + j];
    }
    return loss;
}

// Greedy removal: start from all F; while more than n_f layers are F, turn into S
// the F layer (never layer 0) whose removal gives the smallest proxy loss, the
// lowest layer on ties.
void greedy_pattern(const double* ov, int n, int n_f, char* out) {
    for (int j = 0; j < n; ++j) out[j] = 'F';
    out[n] = '\0';
    for (int nf = n; nf > n_f; --nf) {
        int best = -1;
        double best_loss = 0.0;
        for (int l = 1; l < n; ++l) {
            if (out[l] != 'F') continue;
            out[l] = 'S';
            const double loss = pattern_loss(ov, n, out);
            out[l] = 'F';
            if (best < 0 || loss < best_loss) {
                best = l;
                best_loss = loss;
            }
        }
        out[best] = 'S';
    }
}

}  // namespace dsa
