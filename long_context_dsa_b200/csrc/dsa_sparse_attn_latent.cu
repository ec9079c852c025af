// dsa_sparse_attn_latent.cu -- sparse attention over a shared latent KV row
// (MLA-style: one 576-dim row per token is the key, its first 512 dims the
// value).  Placeholder until the latent kernel lands: reports "no kernel".
#include "dsa_common.cuh"

namespace dsa {

cudaError_t launch_sparse_attn_latent(const void*, const void*, const int*, int, int, int, int, int, float, void*,
                                      bool, WsHeader*, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace dsa
