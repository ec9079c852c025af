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

# (name, n_q, H, d, k, fp8): the first has more work tiles than the array's CTA cap
CASES = [("h32_k2048_3000", 3000, 32, 128, 2048, False),
         ("tiny512", 512, 4, 64, 64, False),
         ("fp8_h64_1100", 1100, 64, 128, 256, True)]


def _inputs(name, L, H, d):
    g = synth.StructuredIndexer("noalloc_" + name, 1, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    return g.layer(0)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry_point_twice(case):
    name, L, H, d, k, fp8 = case
    q, kk, w = _inputs(name, L, H, d)
    qs = ks = None
    dtype = dsa.DSA_BF16
    if fp8:
        q, qs = synth.quantize_e4m3_rows(q)
        kk, ks = synth.quantize_e4m3_rows(kk)
        qs, ks = qs.to(DEV), ks.to(DEV)
        dtype = dsa.DSA_E4M3
    q, kk, w = q.to(DEV), kk.to(DEV), w.to(DEV)
    ref = dsa.idx_score_topk(q, kk, w, k, q_scale=qs, k_scale=ks)
    torch.cuda.synchronize()
    L_ = dsa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for call in range(2):
        out = torch.full((1, L, k), -9, dtype=torch.int32, device=DEV)
        rc = L_.idx_score_topk_noalloc(p(q), p(qs), p(kk), p(ks), p(w), dtype, 1, L, 0, L, H, d, k, p(out), stream)
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
