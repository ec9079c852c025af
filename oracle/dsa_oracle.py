"""Float64 CPU oracle: what the DSA-indexer + IndexCache hot path computes.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.  Plain, slow and
written to be checked against the pages by eye: no blocking, no fusion, no
reordering beyond what each definition states.

Sources (all in Chinese; cited by page title and section):

* [QbitAI] QbitAI article on IndexCache (app.myzaker.com), sections
  "IndexCache" and "GLM-5.2 已经用过了".
* [IndexShare-term] earlyterms.com term page "IndexShare", definition.
* [IndexShare-explainer] "IndexShare 技术解读：4 层共享 indexer 如何把计算成本砍到
  三分之一" (yun88.com), sections "稀疏注意力的隐性开销：indexer" and
  "IndexShare 的共享机制：每 4 层一个 indexer".
* [linkstar] "20万token压进10秒，清华这波操作让AI算力成本直接砍半"
  (linkstar.cloud), sections "长文本的'天价账单'，DSA也躲不过的坑" and
  "'偷懒'的艺术：相邻层其实在重复劳动".

The pages describe the indexer only as "dot product + top-k" ([IndexShare-term],
definition).  This library fixes the DeepSeek-Sparse-Attention lightning-
indexer form

    score[t, s] = sum_h w[t, h] * ReLU(q_I[t, h, :] . k_I[s, :]),   s <= t

and every reading the pages leave open is stated at the function that takes it.

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, brute force on tiny inputs, library routines for special cases and
invariants; none is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "e4m3_decode",
    "indexer_scores",
    "indexer_scores_fp8",
    "topk_select",
    "IndexCache",
    "sparse_attention",
    "layer_group_forward",
    "topk_overlap",
    "check_pattern",
]


# ---------------------------------------------------------------------------
# fp8 e4m3 (OCP 8-bit floating point, "E4M3FN": bias 7, no infinities,
# S.1111.111 is NaN, max finite 448).  Decoding is part of what the fp8
# indexer computes: the kernel reads these bytes, so the oracle must give
# each byte its exact real value.
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Exact float64 value of each OCP E4M3 byte (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    sub = m * 2.0 ** -9                       # e == 0: m/8 * 2^(1-7)
    nrm = (1.0 + m / 8.0) * np.exp2(e - 7.0)  # e >= 1: 1.m * 2^(e-7)
    v = sign * np.where(e == 0, sub, nrm)
    v = np.where((e == 15) & ((c & 7) == 7), np.nan, v)
    return v


def dequantize_e4m3(codes, scale) -> np.ndarray:
    """Real values of per-row scaled E4M3 codes: codes [..., d] (uint8), scale [...]
    (one factor per row); value = e4m3_decode(code) * scale, in float64.  This is the
    fp8 storage the indexer's k_I and q_I use and the fp8 K/V cache: a code times its
    row's scale."""
    return e4m3_decode(codes) * _f64(scale)[..., None]


# ---------------------------------------------------------------------------
# a1: indexer scores
# ---------------------------------------------------------------------------

def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a (CPU) torch tensor of any float dtype."""
    if hasattr(x, "detach"):  # torch tensor; bf16 -> fp64 is exact
        import torch
        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def indexer_scores(q, k, w, q_pos0: int = 0) -> np.ndarray:
    """Causal indexer scores of one sequence, rounded once to float32.

    q: [n_q, H, d] (any float dtype; bf16 values are taken exactly)
    k: [n_kv, d]
    w: [n_q, H]
    Query row i sits at absolute position p = q_pos0 + i and scores keys
    s = 0..p (the token itself included: the pages never exclude it, and
    "k >= t+1 selects every prior token" needs s = t to be a candidate).

    Each score is summed in float64 from the exact inputs and rounded to
    float32 round-to-nearest-even once.  Masked entries (s > p) are -inf.

    [QbitAI] §IndexCache and [linkstar] §DSA: a light indexer in front of
    every attention layer scores the context so that attention sees only
    the chosen tokens; [IndexShare-term]: its work is "dot product + top-k".
    """
    q = _f64(q)
    k = _f64(k)
    w = _f64(w)
    n_q, H, d = q.shape
    n_kv = k.shape[0]
    assert k.shape == (n_kv, d) and w.shape == (n_q, H)
    assert q_pos0 >= 0 and q_pos0 + n_q <= n_kv
    acc = np.zeros((n_q, n_kv), dtype=np.float64)
    for h in range(H):
        dots = q[:, h, :] @ k.T                      # [n_q, n_kv]
        acc += w[:, h:h + 1] * np.maximum(dots, 0.0)  # w[t,h] * ReLU(q.k)
    out = acc.astype(np.float32)
    pos = q_pos0 + np.arange(n_q)[:, None]
    out[np.arange(n_kv)[None, :] > pos] = -np.inf
    return out


def indexer_scores_fp8(q8, q_scale, k8, k_scale, w, q_pos0: int = 0) -> np.ndarray:
    """fp8 indexer: the same score, on the dequantised inputs.

    q8: [n_q, H, d] e4m3 bytes, q_scale: [n_q, H] float32 (> 0)
    k8: [n_kv, d]   e4m3 bytes, k_scale: [n_kv]    float32 (> 0)
    The real value of a quantised element is code_value * its row's scale
    (per-token scaling; the pages are silent on fp8, this is the plain
    reading of "per-token-scaled e4m3").  The score is then exactly
    ``indexer_scores`` of those real values.
    """
    qd = e4m3_decode(q8) * _f64(q_scale)[:, :, None]
    kd = e4m3_decode(k8) * _f64(k_scale)[:, None]
    return indexer_scores(qd, kd, w, q_pos0)


# ---------------------------------------------------------------------------
# a2: per-row top-k
# ---------------------------------------------------------------------------

def topk_select(scores, k: int, q_pos0: int = 0) -> np.ndarray:
    """Top-k token indices per query row, canonical layout.

    scores: float32 [n_q, n_kv]; row i may use columns 0..q_pos0+i.
    Ranking: score descending, then token index ascending (ties go to the
    lower index; -0.0 ranks equal to +0.0).  If the row has p+1 <= k
    candidates, all of them are selected.
    Output: int32 [n_q, k]: the selected indices in ascending order, then
    -1 padding.  The ascending layout is this library's reading (the pages
    fix only the set); it makes set equality byte equality.
    """
    sc = np.asarray(scores, dtype=np.float32)
    n_q, n_kv = sc.shape
    assert k >= 1 and q_pos0 + n_q <= n_kv
    out = np.full((n_q, k), -1, dtype=np.int32)
    for i in range(n_q):
        n = q_pos0 + i + 1
        row = sc[i, :n].astype(np.float64)
        assert np.all(np.isfinite(row)), "scores in the causal range must be finite"
        if n <= k:
            sel = np.arange(n)
        else:
            ids = np.arange(n)
            # primary key: -score (so larger scores first); secondary: index
            order = np.lexsort((ids, -row))
            sel = np.sort(order[:k])
        out[i, :sel.size] = sel
    return out


# ---------------------------------------------------------------------------
# a3 / a5: F/S pattern and the index cache
# ---------------------------------------------------------------------------

def check_pattern(pattern: str) -> None:
    """A layer pattern is a string over {F, S} that starts with F.

    [linkstar] §"'偷懒'的艺术": F layers keep their indexer and cache the
    chosen indices; S layers copy the most recent F layer's cache.
    [QbitAI] §GLM-5.2 and [IndexShare-explainer] §sharing: in groups of four
    the first layer computes, the other three reuse.  A group that starts
    with S has nothing to copy; this library rejects it (reading: the pages
    never start a group with S).
    """
    if not pattern or pattern[0] != "F" or any(c not in "FS" for c in pattern):
        raise ValueError(f"bad layer pattern {pattern!r}: must be over {{F,S}} and start with F")


class IndexCache:
    """One index buffer shared by a layer group.

    An F layer writes its top-k; every later S layer reads exactly that
    array (the same object, so byte-identical), and the cache adds no
    memory beyond the one buffer ([QbitAI] §IndexCache: "不额外占用 GPU 显存").
    """

    def __init__(self):
        self.buf = None
        self.writer = -1

    def put(self, layer: int, idx: np.ndarray) -> None:
        self.buf = idx
        self.writer = layer

    def get(self, layer: int, pattern: str) -> np.ndarray:
        if self.buf is None or self.writer > layer:
            raise ValueError(f"layer {layer} ({pattern[layer]}) has no F layer before it")
        # the most recent F layer at or before `layer` must be the writer
        last_f = max(i for i in range(layer + 1) if pattern[i] == "F")
        if last_f != self.writer:
            raise ValueError("cache writer is not the most recent F layer")
        return self.buf


# ---------------------------------------------------------------------------
# a4: sparse attention over the selected tokens
# ---------------------------------------------------------------------------

def sparse_attention(Q, K, V, idx, scale: float | None = None, d_v: int | None = None) -> np.ndarray:
    """Attention of each query over its selected tokens only, float64.

    Q: [n_q, Hq, d_qk]; K: [n_kv, Hkv, d_qk]; V: [n_kv, Hkv, d_v] or None.
    V=None is the latent (MLA-style) form: one row per token serves as the
    key (all d_qk dims) and as the value (its first d_v dims).
    idx: int [n_q, k]; entries < 0 are skipped.
    Query head h reads KV head g(h) = h // (Hq // Hkv) (grouped-query
    attention; Hq must be a multiple of Hkv).
    scale defaults to 1/sqrt(d_qk) (the pages are silent; plain reading).
    O[t,h] = sum_{j in I[t]} softmax_j(scale * Q[t,h].K[j,g(h)]) V[j,g(h)],
    with the softmax over the valid selected entries, max-subtracted.

    [IndexShare-explainer] §稀疏注意力: each token attends to its top-k
    history tokens only; §sharing: S layers reuse the indices but keep their
    own attention weights, so every layer runs this with its own Q/K/V.
    """
    Q = _f64(Q)
    K = _f64(K)
    n_q, Hq, d_qk = Q.shape
    n_kv, Hkv, d_k2 = K.shape
    assert d_k2 == d_qk and Hq % Hkv == 0
    if V is None:
        assert d_v is not None and d_v <= d_qk
        V = K[:, :, :d_v]
    else:
        V = _f64(V)
    d_v = V.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d_qk)
    gmap = np.arange(Hq) // (Hq // Hkv)
    idx = np.asarray(idx)
    out = np.zeros((n_q, Hq, d_v), dtype=np.float64)
    for i in range(n_q):
        sel = idx[i][idx[i] >= 0].astype(np.int64)
        assert sel.size > 0, "every query must select at least one token"
        Ks = K[sel][:, gmap, :]                       # [m, Hq, d_qk]
        Vs = V[sel][:, gmap, :]                       # [m, Hq, d_v]
        logits = np.einsum("hd,mhd->hm", Q[i], Ks) * scale
        logits -= logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=1, keepdims=True)
        out[i] = np.einsum("hm,mhd->hd", p, Vs)
    return out


# ---------------------------------------------------------------------------
# a5: one layer group
# ---------------------------------------------------------------------------

def sparse_attention_shared(Q, K, V, idx_shared, q_per_idx: int, q_pos0: int, scale: float | None = None,
                            d_v: int | None = None) -> np.ndarray:
    """Several consecutive query tokens reuse one selection (multi-token decode).

    [Term] §IndexShare: the same sharing that lets layers reuse one indexer
    lifts MTP speculative-decoding acceptance.  Reading (the page gives no
    more): query row i (absolute position q_pos0 + i) uses selection row
    i // q_per_idx and, being causal, only the entries of that row at or
    before its own position; then plain sparse attention.
    idx_shared: int [ceil(n_q / q_per_idx), k].
    """
    idx_shared = np.asarray(idx_shared)
    n_q = len(Q)
    rows = []
    for i in range(n_q):
        r = idx_shared[i // q_per_idx].astype(np.int64).copy()
        r[r > q_pos0 + i] = -1
        rows.append(r)
    return sparse_attention(Q, K, V, np.stack(rows), scale=scale, d_v=d_v)


def layer_group_forward(layers, pattern: str, topk: int, q_pos0: int = 0,
                        scale: float | None = None):
    """Run a layer group: F layers index, S layers reuse, all layers attend.

    layers: list of dicts; every layer has Q, K, V (V may be None with d_v
    for the latent form); F layers also have q_I, k_I, w (bf16 indexer) or
    q8, q_scale, k8, k_scale, w (fp8 indexer).
    Returns (idx_per_layer, out_per_layer, indexer_calls).
    idx_per_layer[l] is the very array written by layer l's F layer.

    [QbitAI] §IndexCache: only a few layers keep an indexer, compute top-k
    and cache it; the rest skip it and reuse the most recent result; the
    inference code needs one extra branch.
    """
    check_pattern(pattern)
    assert len(layers) == len(pattern)
    cache = IndexCache()
    idxs, outs, calls = [], [], 0
    for l, (kind, L) in enumerate(zip(pattern, layers)):
        if kind == "F":
            if "q8" in L:
                sc = indexer_scores_fp8(L["q8"], L["q_scale"], L["k8"], L["k_scale"], L["w"], q_pos0)
            else:
                sc = indexer_scores(L["q_I"], L["k_I"], L["w"], q_pos0)
            cache.put(l, topk_select(sc, topk, q_pos0))
            calls += 1
        idx = cache.get(l, pattern)
        idxs.append(idx)
        outs.append(sparse_attention(L["Q"], L["K"], L.get("V"), idx, scale, L.get("d_v")))
    return idxs, outs, calls


# ---------------------------------------------------------------------------
# Overlap of two layers' selections (the motivation for reuse)
# ---------------------------------------------------------------------------

def topk_overlap(idx_a, idx_b, k: int, q_pos0: int = 0) -> float:
    """Mean |I_a[t] & I_b[t]| / k over rows with at least k+1 candidates.

    Rows with p+1 <= k select every token in both layers and are excluded
    (they would be trivially 100%).  [QbitAI] §IndexCache and [linkstar]
    §"'偷懒'的艺术" report 70%-100% for adjacent layers.
    """
    a = np.asarray(idx_a)
    b = np.asarray(idx_b)
    fr = []
    for i in range(a.shape[0]):
        if q_pos0 + i + 1 <= k:
            continue
        fr.append(np.intersect1d(a[i][a[i] >= 0], b[i][b[i] >= 0]).size / k)
    return float(np.mean(fr)) if fr else 1.0


# ---------------------------------------------------------------------------
# F/S pattern search (which layers keep their indexer)
# ---------------------------------------------------------------------------

def overlap_counts(idx_a, idx_b) -> np.ndarray:
    """Per row, the number of token indices (entries >= 0) both selections hold."""
    a = np.asarray(idx_a)
    b = np.asarray(idx_b)
    out = np.zeros(a.shape[0], dtype=np.int64)
    for i in range(a.shape[0]):
        sa = {int(x) for x in a[i] if x >= 0}
        out[i] = sum(1 for x in b[i] if x >= 0 and int(x) in sa)
    return out


def pattern_loss(overlap, pattern: str) -> float:
    """Proxy loss of a pattern: each S layer j loses 1 - overlap[f][j] of its own selection,
    f being the most recent F layer before it (the layer whose indices it reuses)."""
    check_pattern(pattern)
    total, f = 0.0, 0
    for j, c in enumerate(pattern):
        if c == "F":
            f = j
        else:
            total += 1.0 - float(overlap[f][j])
    return total


def pattern_search(overlap, n_f: int) -> str:
    """Greedy F/S choice ([QbitAI] §IndexCache: search which layers to keep by the change in
    loss; [Explainer] §训练无关: a greedy algorithm over calibration data picks the layers).

    Reading: start with every layer F; while more than n_f are F, make S the F layer (not
    layer 0, which must index) whose change raises pattern_loss least, the lowest layer on ties.
    """
    n = len(overlap)
    assert 1 <= n_f <= n
    pat = ["F"] * n
    while pat.count("F") > n_f:
        best, best_loss = None, None
        for l in range(1, n):
            if pat[l] != "F":
                continue
            trial = pat.copy()
            trial[l] = "S"
            loss = pattern_loss(overlap, "".join(trial))
            if best is None or loss < best_loss:
                best, best_loss = l, loss
        pat[best] = "S"
    return "".join(pat)


# ---------------------------------------------------------------------------
# paged caches (serving layout)
# ---------------------------------------------------------------------------

def gather_paged(pool, page_table_row, length: int, page_size: int) -> np.ndarray:
    """Logical cache [length, ...] of one sequence from a page pool [num_pages * page_size, ...]:
    token t sits in row page_table_row[t // page_size] * page_size + t % page_size."""
    pool = np.asarray(pool)
    rows = [int(page_table_row[t // page_size]) * page_size + t % page_size for t in range(length)]
    return pool[rows]
