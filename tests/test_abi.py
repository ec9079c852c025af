"""The C-ABI library loads, exports every declared symbol, and rejects bad
calls on the host before touching a GPU (no compute calls here)."""

import ctypes
import os
import re

import pytest

from long_context_dsa_b200 import dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return sorted(set(re.findall(r"^DSA_API\s+(?:const\s+)?\w+\*?\s+(\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(dsa.LIB_PATH):
        import long_context_dsa_b200.build as b
        b.build()
    return dsa.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(dsa.ABI_SYMBOLS)


def test_version(L):
    assert L.dsa_version() == 100


def test_cache_rejects_null_and_bad_patterns(L):
    c = dsa.IndexCacheStruct()
    assert L.idx_cache_init(None, None, 1, 1) == dsa.DSA_ERR_INVALID_ARG
    assert L.idx_cache_init(ctypes.byref(c), ctypes.c_void_p(0x1000), 4, 8) == dsa.DSA_OK
    out = ctypes.c_void_p(0)
    # nothing written yet
    assert L.idx_cache_get(ctypes.byref(c), 0, b"FSSS", ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG
    assert b"has not written" in L.dsa_last_error()
    for bad in (b"SFFF", b"", b"FXSS", b"fsss"):
        assert L.idx_cache_put(ctypes.byref(c), 0, bad) == dsa.DSA_ERR_INVALID_ARG
    assert L.idx_cache_put(ctypes.byref(c), 1, b"FSSS") == dsa.DSA_ERR_INVALID_ARG  # layer 1 is S
    assert L.idx_cache_put(ctypes.byref(c), 0, b"FSSS") == dsa.DSA_OK
    for layer in range(4):
        out.value = 0
        assert L.idx_cache_get(ctypes.byref(c), layer, b"FSSS", ctypes.byref(out)) == dsa.DSA_OK
        assert out.value == 0x1000  # the same buffer, no copy
    # layer 4 of FSSSFSSS needs F layer 4, which has not written
    assert L.idx_cache_get(ctypes.byref(c), 4, b"FSSSFSSS", ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG
    assert L.idx_cache_get(ctypes.byref(c), 9, b"FSSS", ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG


def test_host_validation_before_any_launch(L):
    v = ctypes.c_void_p(0x1000)
    # GQA needs Hq multiple of Hkv
    assert L.sparse_attn_topk(v, v, v, v, 1, 4, 8, 6, 4, 128, 128, 8, 0.0, v, dsa.DSA_F32, v, 4096,
                              None) == dsa.DSA_ERR_INVALID_ARG
    # unsupported head dim / group size
    assert L.sparse_attn_topk(v, v, v, v, 1, 4, 8, 4, 4, 96, 96, 8, 0.0, v, dsa.DSA_F32, v, 4096,
                              None) == dsa.DSA_ERR_UNSUPPORTED
    assert L.sparse_attn_topk(v, v, v, v, 1, 4, 8, 32, 1, 128, 128, 8, 0.0, v, dsa.DSA_F32, v, 4096,
                              None) == dsa.DSA_ERR_UNSUPPORTED
    n = ctypes.c_size_t(0)
    assert L.idx_topk_scores_workspace_size(4, 0, 8, 0, ctypes.byref(n)) == dsa.DSA_ERR_INVALID_ARG
    assert L.idx_topk_scores_workspace_size(4, 0, 8, 4096, ctypes.byref(n)) == dsa.DSA_ERR_UNSUPPORTED
    assert L.idx_topk_scores_workspace_size(4, 6, 8, 4, ctypes.byref(n)) == dsa.DSA_ERR_INVALID_ARG  # q_pos0+rows > n_kv
    assert L.idx_score_topk_workspace_size(1, 8, 0, 8, 5, 128, 4, dsa.DSA_BF16, ctypes.byref(n)) == dsa.DSA_ERR_UNSUPPORTED
    assert L.idx_score_topk_workspace_size(1, 8, 4, 8, 32, 128, 4, dsa.DSA_BF16, ctypes.byref(n)) == dsa.DSA_ERR_INVALID_ARG
    assert L.idx_score_topk_workspace_size(1, 8, 0, 8, 32, 128, 0, dsa.DSA_BF16, ctypes.byref(n)) == dsa.DSA_ERR_INVALID_ARG
    assert L.idx_score_topk_workspace_size(1, 8, 0, 8, 32, 128, 4, 7, ctypes.byref(n)) == dsa.DSA_ERR_INVALID_ARG


def test_layer_group_rejects_bad_pattern_before_launch(L):
    sh = dsa.group_shape(1, 16, 0, 16, 32, 128, 32, 4, 128, 128, 8)
    c = dsa.IndexCacheStruct()
    assert L.idx_cache_init(ctypes.byref(c), ctypes.c_void_p(0x1000), 16, 8) == dsa.DSA_OK
    layers = (dsa.LayerArgs * 4)()
    st = dsa.GroupStats()
    for pat, n in ((b"SFFF", 4), (b"FSS", 4), (b"FSXS", 4)):
        rc = L.layer_group_forward(ctypes.byref(sh), layers, n, pat, ctypes.byref(c), ctypes.byref(st),
                                   ctypes.c_void_p(0x1000), 1 << 20, None)
        assert rc == dsa.DSA_ERR_INVALID_ARG, pat
    # cache shape mismatch
    c2 = dsa.IndexCacheStruct()
    assert L.idx_cache_init(ctypes.byref(c2), ctypes.c_void_p(0x1000), 8, 8) == dsa.DSA_OK
    rc = L.layer_group_forward(ctypes.byref(sh), layers, 4, b"FSSS", ctypes.byref(c2), ctypes.byref(st),
                               ctypes.c_void_p(0x1000), 1 << 20, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        dsa.idx_topk_scores(torch.zeros(4, 8), 2)
