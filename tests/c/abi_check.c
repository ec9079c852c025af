/* Calls libdsa.so through include/dsa.h from plain C: host-side entry points only (no GPU
 * needed).  Prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "dsa.h"

#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "failed: %s (line %d): %s\n", #cond, __LINE__, \
                    dsa_last_error());                                     \
            return 1;                                                      \
        }                                                                  \
    } while (0)

int main(void) {
    /* greedy F/S search: blocks of layers 0-2, 3-5, 6-7 (0.9 inside a block, 0.3 across) */
    double ov[8 * 8];
    int blk[8] = {0, 0, 0, 1, 1, 1, 2, 2};
    for (int f = 0; f < 8; ++f)
        for (int j = 0; j < 8; ++j) ov[f * 8 + j] = blk[f] == blk[j] ? 0.9 : 0.3;
    char pat[9];
    CHECK(layer_pattern_search(ov, 8, 3, pat) == DSA_OK);
    CHECK(strcmp(pat, "FSSFSSFS") == 0);
    CHECK(layer_pattern_search(ov, 8, 0, pat) == DSA_ERR_INVALID_ARG);
    CHECK(layer_pattern_search(NULL, 8, 3, pat) == DSA_ERR_INVALID_ARG);

    /* index cache: S layers get the F layer's buffer, no launch */
    dsa_index_cache cache;
    int32_t* fake = (int32_t*)(size_t)0x1000;
    CHECK(idx_cache_init(&cache, fake, 16, 8) == DSA_OK);
    const int32_t* got = NULL;
    CHECK(idx_cache_get(&cache, 1, "FSSS", &got) == DSA_ERR_INVALID_ARG); /* nothing written yet */
    CHECK(idx_cache_put(&cache, 0, "FSSS") == DSA_OK);
    CHECK(idx_cache_get(&cache, 3, "FSSS", &got) == DSA_OK && got == fake);
    CHECK(idx_cache_put(&cache, 0, "SFFF") == DSA_ERR_INVALID_ARG);

    /* argument checks that run before any device work */
    void* p = (void*)(size_t)0x1000;
    CHECK(sparse_attn_topk_shared(p, p, p, fake, 1, 4, 0, 8, 8, 8, 64, 64, 8, 0, 0.f, p, DSA_F32, p, 4096,
                                  NULL) == DSA_ERR_INVALID_ARG); /* q_per_idx < 1 */
    CHECK(sparse_attn_topk_shared(p, p, p, fake, 1, 4, 6, 8, 8, 8, 64, 64, 8, 4, 0.f, p, DSA_F32, p, 4096,
                                  NULL) == DSA_ERR_INVALID_ARG); /* positions past the cache */
    CHECK(idx_score_topk_paged(p, p, fake, fake, (const float*)p, 2, 100, 24, 10, 10, 32, 128, 64, fake, p,
                               4096, NULL) == DSA_ERR_INVALID_ARG); /* page size not a power of two */
    CHECK(idx_score_topk_paged(p, p, fake, fake, (const float*)p, 2, 1000, 64, 10, 10, 32, 128, 64, fake, p,
                               4096, NULL) == DSA_ERR_INVALID_ARG); /* table holds 640 < 1000 tokens */
    CHECK(sparse_attn_topk_paged(p, p, p, NULL, fake, fake, 2, 64, 10, 10, 32, 4, 128, 64, 0.f, p, DSA_F32, p,
                                 4096, NULL) == DSA_ERR_INVALID_ARG); /* no page table */
    const float* fs = (const float*)p;
    CHECK(sparse_attn_topk_paged_e4m3(p, p, NULL, p, fs, fake, fake, fake, 2, 64, 10, 10, 32, 4, 128, 64, 0.f, p,
                                      DSA_F32, p, 4096, NULL) == DSA_ERR_INVALID_ARG); /* no K scales */
    CHECK(sparse_attn_topk_paged_e4m3(p, p, fs, p, fs, fake, fake, fake, 2, 64, 10, 10, 32, 4, 96, 64, 0.f, p,
                                      DSA_F32, p, 4096, NULL) == DSA_ERR_UNSUPPORTED); /* d = 96 */
    CHECK(sparse_attn_topk_paged_e4m3(p, p, (const float*)(size_t)0x1002, p, fs, fake, fake, fake, 2, 64, 10, 10,
                                      32, 4, 128, 64, 0.f, p, DSA_F32, p, 4096, NULL)
          == DSA_ERR_INVALID_ARG); /* misaligned scales */
    CHECK(idx_overlap(fake, NULL, 4, 8, fake, NULL) == DSA_ERR_INVALID_ARG);
    CHECK(idx_overlap(fake, fake, 0, 8, fake, NULL) == DSA_ERR_INVALID_ARG);
    size_t n = 0;
    CHECK(idx_score_topk_paged_workspace_size(2, 100, 16, 128, 64, &n) == DSA_ERR_UNSUPPORTED);
    printf("ok\n");
    return 0;
}
