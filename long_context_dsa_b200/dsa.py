"""ctypes binding of libdsa.so (C ABI in include/dsa.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
Functions take torch CUDA tensors (PyTorch supplies device memory and the
current stream) and keep the C entry points' names.  The library is loaded
on first use; if it is missing this raises -- there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_TIMEOUT, DSA_ERR_DEVICE = range(6)
DSA_BF16, DSA_E4M3, DSA_F32 = 0, 1, 2
STATUS_TIMEOUT, STATUS_BAD_INDEX, STATUS_NAN_SCORE, STATUS_OVERFLOW = 1, 2, 4, 8
TOPK_MAX = 2048

ABI_SYMBOLS = (
    "dsa_last_error", "dsa_version", "dsa_check_status", "dsa_reset_status",
    "idx_score_topk_workspace_size", "idx_score_topk", "idx_scores",
    "idx_topk_scores_workspace_size", "idx_topk_scores",
    "idx_cache_init", "idx_cache_put", "idx_cache_get",
    "sparse_attn_topk_workspace_size", "sparse_attn_topk", "sparse_attn_topk_shared",
    "layer_group_forward_workspace_size", "layer_group_forward",
    "idx_score_topk_noalloc", "idx_overlap", "layer_pattern_search",
    "idx_score_topk_paged_workspace_size", "idx_score_topk_paged", "sparse_attn_topk_paged",
    "sparse_attn_topk_paged_e4m3",
)


class DsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[dsa error {code}] {msg}")
        self.code = code


class IndexCacheStruct(ctypes.Structure):
    _fields_ = [("buf", ctypes.c_void_p), ("rows", ctypes.c_int64), ("topk", ctypes.c_int),
                ("writer", ctypes.c_int), ("valid", ctypes.c_int)]


class GroupShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "n_q", "q_pos0", "n_kv", "H_I", "d_I", "idx_dtype",
                                            "Hq", "Hkv", "d_qk", "d_v", "topk")] + \
               [("scale", ctypes.c_float), ("o_dtype", ctypes.c_int)]


class LayerArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_I", "q_scale", "k_I", "k_scale", "w", "Q", "K", "V", "O")]


class GroupStats(ctypes.Structure):
    _fields_ = [("indexer_launches", ctypes.c_int), ("attention_launches", ctypes.c_int),
                ("events", ctypes.POINTER(ctypes.c_void_p))]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdsa.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m long_context_dsa_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, i64, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    psz = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "dsa_last_error": ([], ctypes.c_char_p),
        "dsa_version": ([], i),
        "dsa_check_status": ([vp, vp, ctypes.POINTER(ctypes.c_int)], i),
        "dsa_reset_status": ([vp, vp], i),
        "idx_score_topk_workspace_size": ([i, i, i, i, i, i, i, i, psz], i),
        "idx_score_topk": ([vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp, sz, vp], i),
        "idx_scores": ([vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, vp, sz, vp], i),
        "idx_topk_scores_workspace_size": ([i, i, i, i, psz], i),
        "idx_topk_scores": ([vp, i, i, i, i64, i, vp, vp, sz, vp], i),
        "idx_cache_init": ([ctypes.POINTER(IndexCacheStruct), vp, i64, i], i),
        "idx_cache_put": ([ctypes.POINTER(IndexCacheStruct), i, ctypes.c_char_p], i),
        "idx_cache_get": ([ctypes.POINTER(IndexCacheStruct), i, ctypes.c_char_p, ctypes.POINTER(vp)], i),
        "sparse_attn_topk_workspace_size": ([i, i, i, i, i, i, i, i, psz], i),
        "sparse_attn_topk": ([vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, i, vp, sz, vp], i),
        "sparse_attn_topk_shared": ([vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, f, vp, i, vp, sz, vp], i),
        "layer_group_forward_workspace_size": ([ctypes.POINTER(GroupShape), psz], i),
        "layer_group_forward": ([ctypes.POINTER(GroupShape), ctypes.POINTER(LayerArgs), i, ctypes.c_char_p,
                                 ctypes.POINTER(IndexCacheStruct), ctypes.POINTER(GroupStats), vp, sz, vp], i),
        "idx_score_topk_noalloc": ([vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp], i),
        "idx_overlap": ([vp, vp, i64, i, vp, vp], i),
        "idx_score_topk_paged_workspace_size": ([i, i, i, i, i, psz], i),
        "idx_score_topk_paged": ([vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp, sz, vp], i),
        "sparse_attn_topk_paged": ([vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, i, vp, sz, vp], i),
        "sparse_attn_topk_paged_e4m3": ([vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, i, vp, sz,
                                         vp], i),
        "layer_pattern_search": ([ctypes.POINTER(ctypes.c_double), i, i, ctypes.c_char_p], i),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(rc: int):
    if rc != DSA_OK:
        raise DsaError(rc, lib().dsa_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor (got {t.dtype}, {t.device})")


def _workspace(nbytes: int, device) -> torch.Tensor:
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def read_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the workspace status word; return its DSA_STATUS_* bits."""
    bits = ctypes.c_int(0)
    rc = lib().dsa_check_status(_ptr(workspace), _stream(stream), ctypes.byref(bits))
    if rc not in (DSA_OK, DSA_ERR_TIMEOUT, DSA_ERR_DEVICE):
        raise DsaError(rc, lib().dsa_last_error().decode(errors="replace"))
    return bits.value


def check_status(workspace: torch.Tensor, stream=None) -> None:
    """Synchronise, read and clear the workspace status word; raise DsaError if a kernel flagged an error."""
    bits = ctypes.c_int(0)
    rc = lib().dsa_check_status(_ptr(workspace), _stream(stream), ctypes.byref(bits))
    if rc != DSA_OK:
        raise DsaError(rc, lib().dsa_last_error().decode(errors="replace"))


# ------------------------------------------------------------------ indexer
def _idx_dtype(q_I):
    if q_I.dtype == torch.bfloat16:
        return DSA_BF16
    if q_I.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_E4M3
    raise ValueError("q_I must be bf16 or e4m3 (uint8 codes)")


def _idx_dims(q_I, k_I, q_pos0):
    if q_I.dim() != 4 or k_I.dim() != 3:
        raise ValueError("q_I is [B, n_q, H_I, d_I] and k_I is [B, n_kv, d_I]")
    B, n_q, H, d = q_I.shape
    n_kv = k_I.shape[1]
    if k_I.shape[0] != B or k_I.shape[2] != d:
        raise ValueError("k_I shape does not match q_I")
    return B, n_q, H, d, n_kv


def idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype=DSA_BF16) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H_I, d_I, topk, dtype, ctypes.byref(n)))
    return n.value


def idx_score_topk(q_I, k_I, w, topk: int, q_pos0: int = 0, q_scale=None, k_scale=None,
                   out=None, workspace=None, stream=None) -> torch.Tensor:
    """Fused indexer scores + per-row top-k -> int32 [B, n_q, topk] (ascending, -1 padded)."""
    dt = _idx_dtype(q_I)
    B, n_q, H, d, n_kv = _idx_dims(q_I, k_I, q_pos0)
    for t, n in ((q_I, "q_I"), (k_I, "k_I")):
        _need(t, q_I.dtype, n)
    _need(w, torch.float32, "w")
    if dt == DSA_E4M3:
        _need(q_scale, torch.float32, "q_scale")
        _need(k_scale, torch.float32, "k_scale")
    if out is None:
        out = torch.empty((B, n_q, topk), dtype=torch.int32, device=q_I.device)
    _need(out, torch.int32, "out")
    if workspace is None:
        workspace = _workspace(idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H, d, topk, dt), q_I.device)
    _check(lib().idx_score_topk(_ptr(q_I), _ptr(q_scale), _ptr(k_I), _ptr(k_scale), _ptr(w), dt, B, n_q, q_pos0,
                                n_kv, H, d, topk, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def idx_scores(q_I, k_I, w, q_pos0: int = 0, q_scale=None, k_scale=None, out=None, workspace=None,
               stream=None) -> torch.Tensor:
    """Indexer scores without selection (test/debug) -> fp32 [B, n_q, n_kv]; unvisited entries keep `out`'s values."""
    dt = _idx_dtype(q_I)
    B, n_q, H, d, n_kv = _idx_dims(q_I, k_I, q_pos0)
    _need(w, torch.float32, "w")
    if out is None:
        out = torch.full((B, n_q, n_kv), float("nan"), dtype=torch.float32, device=q_I.device)
    _need(out, torch.float32, "out")
    if workspace is None:
        workspace = _workspace(256, q_I.device)
    _check(lib().idx_scores(_ptr(q_I), _ptr(q_scale), _ptr(k_I), _ptr(k_scale), _ptr(w), dt, B, n_q, q_pos0, n_kv,
                            H, d, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def idx_topk_scores(scores, topk: int, q_pos0: int = 0, n_kv: int | None = None, out=None, workspace=None,
                    stream=None) -> torch.Tensor:
    """Top-k selection alone on fp32 scores [rows, ld] -> int32 [rows, topk]."""
    _need(scores, torch.float32, "scores")
    rows, ld = scores.shape
    n_kv = ld if n_kv is None else n_kv
    if out is None:
        out = torch.empty((rows, topk), dtype=torch.int32, device=scores.device)
    _need(out, torch.int32, "out")
    if workspace is None:
        n = ctypes.c_size_t(0)
        _check(lib().idx_topk_scores_workspace_size(rows, q_pos0, n_kv, topk, ctypes.byref(n)))
        workspace = _workspace(n.value, scores.device)
    _check(lib().idx_topk_scores(_ptr(scores), rows, q_pos0, n_kv, ld, topk, _ptr(out), _ptr(workspace),
                                 workspace.numel(), _stream(stream)))
    return out


# -------------------------------------------------------------- index cache
class IndexCache:
    """Host descriptor around one int32 [rows, topk] device buffer (the group's index cache)."""

    def __init__(self, buf: torch.Tensor):
        _need(buf, torch.int32, "buf")
        self.buf = buf
        self.c = IndexCacheStruct()
        rows = buf.numel() // buf.shape[-1]
        _check(lib().idx_cache_init(ctypes.byref(self.c), _ptr(buf), rows, buf.shape[-1]))

    def put(self, layer: int, pattern: str):
        _check(lib().idx_cache_put(ctypes.byref(self.c), layer, pattern.encode()))

    def get_ptr(self, layer: int, pattern: str) -> int:
        p = ctypes.c_void_p(0)
        _check(lib().idx_cache_get(ctypes.byref(self.c), layer, pattern.encode(), ctypes.byref(p)))
        return p.value


def idx_cache_get(cache: IndexCache, layer: int, pattern: str) -> torch.Tensor:
    """The index tensor layer `layer` uses: the cache buffer itself (no copy, no launch)."""
    ptr = cache.get_ptr(layer, pattern)
    assert ptr == cache.buf.data_ptr()
    return cache.buf


# --------------------------------------------------------- sparse attention
def sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk, ctypes.byref(n)))
    return n.value


def sparse_attn_topk(Q, K, V, idx, scale: float | None = None, o_dtype=torch.float32, d_v: int | None = None,
                     out=None, workspace=None, stream=None) -> torch.Tensor:
    """O[b,i,h] = softmax over idx[b,i] of scale*Q.K, times V -> [B, n_q, Hq, d_v]."""
    _need(Q, torch.bfloat16, "Q")
    _need(K, torch.bfloat16, "K")
    if V is not None:
        _need(V, torch.bfloat16, "V")
    _need(idx, torch.int32, "idx")
    B, n_q, Hq, d_qk = Q.shape
    n_kv, Hkv = K.shape[1], K.shape[2]
    if V is not None:
        d_v = V.shape[3]
    elif d_v is None:
        raise ValueError("latent form (V=None) needs d_v")
    topk = idx.shape[-1]
    od = DSA_F32 if o_dtype == torch.float32 else DSA_BF16
    if out is None:
        out = torch.empty((B, n_q, Hq, d_v), dtype=o_dtype, device=Q.device)
    _need(out, o_dtype, "out")
    if workspace is None:
        workspace = _workspace(sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk), Q.device)
    _check(lib().sparse_attn_topk(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk,
                                  float(scale or 0.0), _ptr(out), od, _ptr(workspace), workspace.numel(),
                                  _stream(stream)))
    return out


def sparse_attn_topk_shared(Q, K, V, idx, q_per_idx: int, q_pos0: int, scale: float | None = None,
                            o_dtype=torch.float32, d_v: int | None = None, out=None, workspace=None,
                            stream=None) -> torch.Tensor:
    """As sparse_attn_topk, but query row i uses index row idx[b, i // q_per_idx], causally limited to
    its own position q_pos0 + i.  idx: [B, ceil(n_q / q_per_idx), topk]."""
    _need(Q, torch.bfloat16, "Q")
    _need(K, torch.bfloat16, "K")
    if V is not None:
        _need(V, torch.bfloat16, "V")
    _need(idx, torch.int32, "idx")
    B, n_q, Hq, d_qk = Q.shape
    n_kv, Hkv = K.shape[1], K.shape[2]
    if V is not None:
        d_v = V.shape[3]
    elif d_v is None:
        raise ValueError("latent form (V=None) needs d_v")
    if idx.shape[1] != (n_q + q_per_idx - 1) // q_per_idx:
        raise ValueError("idx must have ceil(n_q / q_per_idx) rows per sequence")
    topk = idx.shape[-1]
    od = DSA_F32 if o_dtype == torch.float32 else DSA_BF16
    if out is None:
        out = torch.empty((B, n_q, Hq, d_v), dtype=o_dtype, device=Q.device)
    _need(out, o_dtype, "out")
    if workspace is None:
        workspace = _workspace(sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d_qk, d_v, topk), Q.device)
    _check(lib().sparse_attn_topk_shared(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), B, n_q, q_pos0, n_kv, Hq, Hkv, d_qk,
                                         d_v, topk, q_per_idx, float(scale or 0.0), _ptr(out), od, _ptr(workspace),
                                         workspace.numel(), _stream(stream)))
    return out


# -------------------------------------------------------------- paged decode
def idx_score_topk_paged(q_I, k_pages, page_table, seq_lens, w, topk: int, max_seq_len: int, out=None,
                         workspace=None, stream=None) -> torch.Tensor:
    """One query per sequence over a paged key cache: q_I [B, H, d], k_pages [num_pages, page_size, d],
    page_table [B, max_pages], seq_lens [B] (int32, device) -> idx [B, topk]."""
    _need(q_I, torch.bfloat16, "q_I")
    _need(k_pages, torch.bfloat16, "k_pages")
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    _need(w, torch.float32, "w")
    B, H, d = q_I.shape
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    max_pages = page_table.shape[1]
    if out is None:
        out = torch.empty((B, topk), dtype=torch.int32, device=q_I.device)
    if workspace is None:
        n = ctypes.c_size_t(0)
        _check(lib().idx_score_topk_paged_workspace_size(B, max_seq_len, H, d, topk, ctypes.byref(n)))
        workspace = _workspace(n.value, q_I.device)
    _check(lib().idx_score_topk_paged(_ptr(q_I), _ptr(k_pages), _ptr(page_table), _ptr(seq_lens), _ptr(w), B,
                                      max_seq_len, page_size, num_pages, max_pages, H, d, topk, _ptr(out),
                                      _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def idx_score_topk_paged_workspace_size(B, max_seq_len, H, d, topk) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().idx_score_topk_paged_workspace_size(B, max_seq_len, H, d, topk, ctypes.byref(n)))
    return n.value


def sparse_attn_topk_paged(Q, K_pages, V_pages, page_table, seq_lens, idx, scale: float | None = None,
                           o_dtype=torch.float32, out=None, workspace=None, stream=None) -> torch.Tensor:
    """Q [B, Hq, d]; K_pages, V_pages [num_pages, page_size, Hkv, d]; idx [B, topk] -> O [B, Hq, d]."""
    for t, n in ((Q, "Q"), (K_pages, "K_pages"), (V_pages, "V_pages")):
        _need(t, torch.bfloat16, n)
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    _need(idx, torch.int32, "idx")
    B, Hq, d = Q.shape
    num_pages, page_size, Hkv = K_pages.shape[0], K_pages.shape[1], K_pages.shape[2]
    max_pages = page_table.shape[1]
    topk = idx.shape[-1]
    od = DSA_F32 if o_dtype == torch.float32 else DSA_BF16
    if out is None:
        out = torch.empty((B, Hq, d), dtype=o_dtype, device=Q.device)
    if workspace is None:
        workspace = _workspace(sparse_attn_topk_workspace_size(B, 1, num_pages * page_size, Hq, Hkv, d, d, topk),
                               Q.device)
    _check(lib().sparse_attn_topk_paged(_ptr(Q), _ptr(K_pages), _ptr(V_pages), _ptr(page_table), _ptr(seq_lens),
                                        _ptr(idx), B, page_size, num_pages, max_pages, Hq, Hkv, d, topk,
                                        float(scale or 0.0), _ptr(out), od, _ptr(workspace), workspace.numel(),
                                        _stream(stream)))
    return out


def sparse_attn_topk_paged_e4m3(Q, K8_pages, k_scale, V8_pages, v_scale, page_table, seq_lens, idx,
                                scale: float | None = None, o_dtype=torch.float32, out=None, workspace=None,
                                stream=None) -> torch.Tensor:
    """sparse_attn_topk_paged over an fp8 cache: K8_pages, V8_pages [num_pages, page_size, Hkv, d]
    E4M3 codes (uint8), k_scale, v_scale [num_pages, page_size, Hkv] fp32 (real row = code x scale)."""
    _need(Q, torch.bfloat16, "Q")
    for t, n in ((K8_pages, "K8_pages"), (V8_pages, "V8_pages")):
        _need(t, torch.uint8, n)
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, torch.float32, n)
    _need(page_table, torch.int32, "page_table")
    _need(seq_lens, torch.int32, "seq_lens")
    _need(idx, torch.int32, "idx")
    B, Hq, d = Q.shape
    num_pages, page_size, Hkv = K8_pages.shape[0], K8_pages.shape[1], K8_pages.shape[2]
    if tuple(k_scale.shape) != (num_pages, page_size, Hkv) or tuple(v_scale.shape) != (num_pages, page_size, Hkv):
        raise ValueError("scales must be [num_pages, page_size, Hkv]")
    max_pages = page_table.shape[1]
    topk = idx.shape[-1]
    od = DSA_F32 if o_dtype == torch.float32 else DSA_BF16
    if out is None:
        out = torch.empty((B, Hq, d), dtype=o_dtype, device=Q.device)
    if workspace is None:
        workspace = _workspace(sparse_attn_topk_workspace_size(B, 1, num_pages * page_size, Hq, Hkv, d, d, topk),
                               Q.device)
    _check(lib().sparse_attn_topk_paged_e4m3(_ptr(Q), _ptr(K8_pages), _ptr(k_scale), _ptr(V8_pages), _ptr(v_scale),
                                             _ptr(page_table), _ptr(seq_lens), _ptr(idx), B, page_size, num_pages,
                                             max_pages, Hq, Hkv, d, topk, float(scale or 0.0), _ptr(out), od,
                                             _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


# -------------------------------------------------------------- F/S pattern search
def idx_overlap(idx_a: torch.Tensor, idx_b: torch.Tensor, counts=None, stream=None) -> torch.Tensor:
    """Per-row |A ∩ B| of two canonical index buffers [..., topk] (int32 counts, one per row)."""
    _need(idx_a, torch.int32, "idx_a")
    _need(idx_b, torch.int32, "idx_b")
    if idx_a.shape != idx_b.shape:
        raise ValueError("index buffers differ in shape")
    topk = idx_a.shape[-1]
    rows = idx_a.numel() // topk
    if counts is None:
        counts = torch.empty(rows, dtype=torch.int32, device=idx_a.device)
    _check(lib().idx_overlap(_ptr(idx_a), _ptr(idx_b), rows, topk, _ptr(counts), _stream(stream)))
    return counts


def layer_pattern_search(overlap, n_f: int) -> str:
    """Greedy F/S pattern with n_f F layers from a host [n_layers, n_layers] overlap matrix."""
    import numpy as np

    ov = np.ascontiguousarray(np.asarray(overlap, dtype=np.float64))
    n = ov.shape[0]
    if ov.shape != (n, n):
        raise ValueError("overlap must be square")
    buf = ctypes.create_string_buffer(n + 1)
    _check(lib().layer_pattern_search(ov.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), n, n_f, buf))
    return buf.value.decode()


# -------------------------------------------------------------- layer group
def group_shape(B, n_q, q_pos0, n_kv, H_I, d_I, Hq, Hkv, d_qk, d_v, topk, idx_dtype=DSA_BF16, scale=0.0,
                o_dtype=DSA_F32) -> GroupShape:
    return GroupShape(B, n_q, q_pos0, n_kv, H_I, d_I, idx_dtype, Hq, Hkv, d_qk, d_v, topk, scale, o_dtype)


def layer_group_forward_workspace_size(shape: GroupShape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().layer_group_forward_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def layer_group_forward(shape: GroupShape, layers, pattern: str, cache: IndexCache, workspace=None,
                        stream=None, events=None) -> GroupStats:
    """Run one layer group.  `layers`: list of dicts with Q, K, V (or None), O and, on F layers,
    q_I, k_I, w (+ q_scale, k_scale for e4m3).  `events`: optional list of 3*len(layers)
    torch.cuda.Event (already recorded once) that the library records around each launch.
    Returns the host launch counters."""
    arr = (LayerArgs * len(layers))()
    for a, L in zip(arr, layers):
        for name in ("q_I", "q_scale", "k_I", "k_scale", "w", "Q", "K", "V", "O"):
            t = L.get(name)
            setattr(a, name, None if t is None else t.data_ptr())
    if workspace is None:
        workspace = _workspace(layer_group_forward_workspace_size(shape), layers[0]["Q"].device)
    stats = GroupStats()
    if events is not None:
        if len(events) != 3 * len(layers):
            raise ValueError("events must hold 3 per layer")
        handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        stats.events = ctypes.cast(handles, ctypes.POINTER(ctypes.c_void_p))
    _check(lib().layer_group_forward(ctypes.byref(shape), arr, len(layers), pattern.encode(), ctypes.byref(cache.c),
                                     ctypes.byref(stats), _ptr(workspace), workspace.numel(), _stream(stream)))
    return stats


# ------------------------------------------------- no-allocation variant
def idx_score_topk_noalloc(q_I, k_I, w, topk: int, q_pos0: int = 0, q_scale=None, k_scale=None,
                           out=None, stream=None) -> torch.Tensor:
    """idx_score_topk without a workspace, for callers that cannot allocate device memory
    (e.g. code running inside another runtime's memory pool).  Scratch lives in a fixed
    32 MiB array inside the library; calls must not overlap on the GPU.  `out` should be
    passed by such callers (allocating it here is only a convenience for tests)."""
    dt = _idx_dtype(q_I)
    B, n_q, H, d, n_kv = _idx_dims(q_I, k_I, q_pos0)
    for t, n in ((q_I, "q_I"), (k_I, "k_I")):
        _need(t, q_I.dtype, n)
    _need(w, torch.float32, "w")
    if out is None:
        out = torch.empty((B, n_q, topk), dtype=torch.int32, device=q_I.device)
    _need(out, torch.int32, "out")
    _check(lib().idx_score_topk_noalloc(_ptr(q_I), _ptr(q_scale), _ptr(k_I), _ptr(k_scale), _ptr(w), dt, B, n_q,
                                        q_pos0, n_kv, H, d, topk, _ptr(out), _stream(stream)))
    return out
