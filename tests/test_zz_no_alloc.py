"""The no-allocation indexer entry point (idx_score_topk_noalloc).

Some callers cannot allocate device memory -- code running inside another
runtime's memory pool, or on a path that must never call cudaMalloc -- so
they cannot pass the workspace idx_score_topk needs.  idx_score_topk_noalloc
serves them from a fixed scratch array inside the library.  This test calls
it through the C ABI twice in a row (the second call reuses the array with
the first call's contents still in it) and checks both outputs against the
workspace entry point on the same inputs.  The file is named to be collected
last so a run that stops at the first failure has run every other test.
"""

import ctypes

import pytest
import torch

from long_context_dsa_b200 import dsa, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (name, B, n_q, n_kv, H, d, k, fp8): the first has more work tiles than the array's CTA cap; the
# decode case (one query per sequence at the end of its cache) takes the split decode kernel,
# whose score keys, histograms and bin-select scratch also live in the array
CASES = [("h32_k2048_3000", 1, 3000, 3000, 32, 128, 2048, False),
         ("tiny512", 1, 512, 512, 4, 64, 64, False),
         ("fp8_h64_1100", 1, 1100, 1100, 64, 128, 256, True),
         ("decode_b8_4096", 8, 1, 4096, 32, 128, 2048, False)]


def _inputs(name, B, n_q, L, H, d):
    g = synth.StructuredIndexer("noalloc_" + name, B, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    if n_q == L:
        return g.layer(0)
    q, w = g.queries(0, L - n_q, L)
    return q, g.keys(0), w


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry_point_twice(case):
    name, B, n_q, L, H, d, k, fp8 = case
    q_pos0 = L - n_q
    q, kk, w = _inputs(name, B, n_q, L, H, d)
    qs = ks = None
    dtype = dsa.DSA_BF16
    if fp8:
        q, qs = synth.quantize_e4m3_rows(q)
        kk, ks = synth.quantize_e4m3_rows(kk)
        qs, ks = qs.to(DEV), ks.to(DEV)
        dtype = dsa.DSA_E4M3
    q, kk, w = q.to(DEV), kk.to(DEV), w.to(DEV)
    ref = dsa.idx_score_topk(q, kk, w, k, q_pos0=q_pos0, q_scale=qs, k_scale=ks)
    torch.cuda.synchronize()
    L_ = dsa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for call in range(2):
        out = torch.full((B, n_q, k), -9, dtype=torch.int32, device=DEV)
        rc = L_.idx_score_topk_noalloc(p(q), p(qs), p(kk), p(ks), p(w), dtype, B, n_q, q_pos0, L, H, d, k, p(out),
                                       stream)
        assert rc == dsa.DSA_OK, L_.dsa_last_error()
        torch.cuda.synchronize()
        # same kernel arithmetic as the workspace path: the selections agree exactly
        assert torch.equal(out, ref), f"call {call}: differs from idx_score_topk"


def test_noalloc_rejects_bad_arguments():
    L_ = dsa.lib()
    v = ctypes.c_void_p(0x1000)
    assert L_.idx_score_topk_noalloc(v, None, v, None, v, dsa.DSA_BF16, 1, 8, 0, 8, 32, 128, 0, v, None) \
        == dsa.DSA_ERR_INVALID_ARG
    assert L_.idx_score_topk_noalloc(v, None, v, None, v, dsa.DSA_BF16, 1, 8, 0, 8, 32, 128, 4096, v, None) \
        == dsa.DSA_ERR_UNSUPPORTED
