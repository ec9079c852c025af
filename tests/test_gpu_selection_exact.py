"""Every selection path of the library, byte for byte against the oracle.

The inputs are integers (q_I, k_I) and multiples of 1/4 (w), so every indexer score is
exact in fp32 whatever order the sums run in (``synth.integer_indexer``): the GPU's scores
equal the oracle's bit for bit, and the selection rule (k largest, ties to the lower token
index, ascending output, -1 padding) leaves exactly one correct answer.  Small value
ranges make equal scores and zero scores common, so tie-breaking, the streaming prune of
the fused kernel (and its exact fallback when one score value holds more ties than the
prune's slack) and the bin select of one-query decode (histogram of the score keys' top
bits, kept keys, exact select; whole-row select when the kept keys overflow), over
contiguous and paged caches, are all checked for exactness, not within a tolerance.

[QbitAI] §IndexCache / [Term] "dot product + top-k": the selection is the k best scores
of each query row; ties to the lower index is this library's stated rule.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _expect_identical(gpu_idx, ora_idx, what):
    gpu_idx = np.asarray(gpu_idx)
    bad = np.nonzero(~np.all(gpu_idx == ora_idx, axis=-1))[0]
    assert bad.size == 0, (f"{what}: {bad.size} of {gpu_idx.shape[0]} rows differ from the oracle, "
                           f"first row {bad[0]}")


def _run_fused(q, k, w, topk, q_pos0=0, q_scale=None, k_scale=None):
    B, n_q, H, d = q.shape
    n_kv = k.shape[1]
    dt = dsa.DSA_E4M3 if q.dtype == torch.uint8 else dsa.DSA_BF16
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H, d, topk, dt), dtype=torch.uint8,
                     device=DEV)
    idx = dsa.idx_score_topk(q.to(DEV), k.to(DEV), w.to(DEV), topk, q_pos0=q_pos0,
                             q_scale=None if q_scale is None else q_scale.to(DEV),
                             k_scale=None if k_scale is None else k_scale.to(DEV), workspace=ws)
    assert dsa.read_status(ws) == 0
    return idx.cpu().numpy()


# (name, B, n_q, q_pos0, n_kv, H, d, topk, lo, hi)
PREFILL = [
    # the 200K workload's head shape with top-2048: rows past t = 2047 prune while streaming
    ("h32_k2048", 1, 5000, 0, 5000, 32, 128, 2048, -4, 4),
    # values in {-1, 0, 1}: a handful of distinct scores, so one value holds far more ties than
    # the prune's k/8 slack and the exact radix fallback must split them by index
    ("ties_h32_k512", 1, 4000, 0, 4000, 32, 128, 512, -1, 1),
    # the 16K workload's head shape, many prunes at a small top-k
    ("h64_k256", 1, 3000, 0, 3000, 64, 128, 256, -4, 4),
    ("h64_k1", 1, 700, 0, 700, 64, 128, 1, -2, 2),
    ("h16_k100", 1, 1300, 0, 1300, 16, 128, 100, -3, 3),
    ("h8_k64", 1, 900, 0, 900, 8, 128, 64, -3, 3),
    ("h4d64_k64", 1, 2000, 0, 2000, 4, 64, 64, -4, 4),
    # a later chunk of a chunked prefill, two sequences, ragged query tile
    ("chunk_b2", 2, 300, 700, 1000, 64, 128, 128, -3, 3),
]


@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_fused_prefill_selection_is_exact(case):
    name, B, n_q, q_pos0, n_kv, H, d, topk, lo, hi = case
    q, k, w = synth.integer_indexer(name, B, n_kv, H, d, lo, hi)
    q = q[:, q_pos0:q_pos0 + n_q].contiguous()
    w = w[:, q_pos0:q_pos0 + n_q].contiguous()
    idx = _run_fused(q, k, w, topk, q_pos0)
    for b in range(B):
        ora = oracle.topk_select(oracle.indexer_scores(q[b], k[b], w[b], q_pos0), topk, q_pos0)
        _expect_identical(idx[b], ora, f"{name} b={b}")


def test_fused_selection_with_survivors_in_one_lane_range_is_exact():
    """Keys at positions s mod 128 < 32 (one epilogue warp's lanes) are doubled, so that warp's
    share of each candidate buffer fills first and the prune has to rebalance the shares."""
    B, L, H, d, topk = 1, 6000, 32, 128, 2048
    q, k, w = synth.integer_indexer("skew", B, L, H, d, -4, 4)
    hot = (torch.arange(L) % 128) < 32
    k = k.float()
    k[:, hot] *= 2.0
    k = k.to(torch.bfloat16)
    idx = _run_fused(q, k, w, topk)
    ora = oracle.topk_select(oracle.indexer_scores(q[0], k[0], w[0]), topk)
    _expect_identical(idx[0], ora, "skewed lanes")


def test_all_equal_scores_select_the_first_tokens():
    """Zero queries give every key the score 0: each row must select tokens 0..k-1."""
    B, L, H, d, topk = 1, 3000, 32, 128, 1000
    _, k, w = synth.integer_indexer("zeros", B, L, H, d, -4, 4)
    q = torch.zeros((B, L, H, d), dtype=torch.bfloat16)
    idx = _run_fused(q, k, w, topk)[0]
    for t in (0, 999, 1000, 2999):
        n = min(topk, t + 1)
        assert np.array_equal(idx[t, :n], np.arange(n)) and np.all(idx[t, n:] == -1), t


def test_fused_fp8_selection_is_exact():
    B, L, H, d, topk = 1, 3000, 64, 128, 512
    q8, qs, k8, ks, w = synth.integer_indexer_e4m3("fp8x", B, L, H, d, -3, 3)
    idx = _run_fused(q8, k8, w, topk, q_scale=qs, k_scale=ks)
    ora = oracle.topk_select(oracle.indexer_scores_fp8(q8[0].numpy(), qs[0].numpy(), k8[0].numpy(),
                                                       ks[0].numpy(), w[0]), topk)
    _expect_identical(idx[0], ora, "fp8 prefill")


def _decode_case(name, B, n_kv, H, topk, lo, hi, fp8=False):
    """One query per sequence at the end of an n_kv-token cache (the split decode kernel)."""
    d = 128
    if fp8:
        q, qs, k, ks, w = synth.integer_indexer_e4m3(name, B, n_kv, H, d, lo, hi, q_rows=1)
        idx = _run_fused(q, k, w, topk, q_pos0=n_kv - 1, q_scale=qs, k_scale=ks)
        for b in range(B):
            sc = oracle.indexer_scores_fp8(q[b].numpy(), qs[b].numpy(), k[b].numpy(), ks[b].numpy(), w[b],
                                           n_kv - 1)
            _expect_identical(idx[b], oracle.topk_select(sc, topk, n_kv - 1), f"{name} b={b}")
        return
    q, k, w = synth.integer_indexer(name, B, n_kv, H, d, lo, hi, q_rows=1)
    idx = _run_fused(q, k, w, topk, q_pos0=n_kv - 1)
    for b in range(B):
        sc = oracle.indexer_scores(q[b], k[b], w[b], n_kv - 1)
        _expect_identical(idx[b], oracle.topk_select(sc, topk, n_kv - 1), f"{name} b={b}")


@pytest.mark.parametrize("case", [
    # (name, B, n_kv, H, topk, lo, hi): one query per sequence, the bin select
    ("dec_b4_h32", 4, 20000, 32, 2048, -4, 4),
    ("dec_b2_h64_ties", 2, 9000, 64, 2048, -1, 1),
    ("dec_b8_h32_k300", 8, 4100, 32, 300, -3, 3),
], ids=lambda c: c[0])
def test_decode_selection_is_exact(case):
    _decode_case(*case)


def test_decode_fp8_selection_is_exact():
    _decode_case("dec_fp8_b3", 3, 12000, 64, 2048, -3, 3, fp8=True)


def test_decode_long_cache_selection_is_exact():
    """One query against a 1.7M-token cache: the score keys of the whole row go through the
    bin select (or, with these heavily tied scores, its whole-row fallback)."""
    _decode_case("dec_long", 1, 1_700_000, 32, 2048, -2, 2)


def _bin_select_stats(ws):
    """(rows selected from the whole row, most keys a row kept) recorded by the decode bin select."""
    v = ws[12:20].cpu().view(torch.int32).tolist()
    return v[0], v[1]


def _decode_with_stats(name, B, n_kv, H, topk, lo, hi):
    d = 128
    q, k, w = synth.integer_indexer(name, B, n_kv, H, d, lo, hi, q_rows=1)
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, 1, n_kv - 1, n_kv, H, d, topk, dsa.DSA_BF16),
                     dtype=torch.uint8, device=DEV)
    idx = dsa.idx_score_topk(q.to(DEV), k.to(DEV), w.to(DEV), topk, q_pos0=n_kv - 1, workspace=ws)
    assert dsa.read_status(ws) == 0
    idx = idx.cpu().numpy()
    for b in range(B):
        sc = oracle.indexer_scores(q[b], k[b], w[b], n_kv - 1)
        _expect_identical(idx[b], oracle.topk_select(sc, topk, n_kv - 1), f"{name} b={b}")
    return _bin_select_stats(ws)


def test_decode_bin_select_fast_path_and_whole_row_fallback_are_exact():
    """The decode select keeps the keys of the k-th key's histogram bin and above and selects
    among them; spread scores take that path, while equal scores (every key in one bin) overflow
    the kept-key buffers and are selected from the whole row.  Both must match the oracle."""
    full, kept = _decode_with_stats("bin_fast", 3, 30000, 32, 512, -8, 8)
    assert full == 0 and 512 <= kept <= 16384, (full, kept)
    full, kept = _decode_with_stats("bin_equal", 2, 30000, 32, 512, 0, 0)
    assert full == 2, (full, kept)


def test_paged_decode_long_sequence_selection_is_exact():
    """A paged sequence of 1.7M tokens in shuffled pages: its score keys and histogram, then the
    bin select (with these heavily tied scores, its whole-row select)."""
    n, P, H, d, topk = 1_700_000, 256, 32, 128, 2048
    q, k, w = synth.integer_indexer("paged_stream", 1, n, H, d, -2, 2, q_rows=1)
    pages = (n + P - 1) // P
    perm = np.random.default_rng(5).permutation(pages).astype(np.int32)
    pool = torch.zeros((pages * P, d), dtype=torch.bfloat16)
    pool.view(pages, P, d)[torch.from_numpy(perm).long()] = torch.cat(
        [k[0], torch.zeros((pages * P - n, d), dtype=torch.bfloat16)]).view(pages, P, d)
    table = torch.from_numpy(perm[None]).to(DEV)
    ws = torch.zeros(dsa.idx_score_topk_paged_workspace_size(1, n, H, d, topk), dtype=torch.uint8, device=DEV)
    idx = dsa.idx_score_topk_paged(q[:, 0].contiguous().to(DEV), pool.view(pages, P, d).to(DEV), table,
                                   torch.tensor([n], dtype=torch.int32, device=DEV), w[:, 0].contiguous().to(DEV),
                                   topk, n, workspace=ws)
    assert dsa.read_status(ws) == 0
    sc = oracle.indexer_scores(q[0], k[0], w[0], n - 1)
    _expect_identical(idx.cpu().numpy(), oracle.topk_select(sc, topk, n - 1), "paged 1.7M")


def test_paged_decode_selection_is_exact():
    lens = [1, 100, 1500, 3000, 4097]
    P, H, d, topk = 64, 32, 128, 512
    B, Lmax = len(lens), max(lens)
    q_all, k, w_all = synth.integer_indexer("paged_exact", B, Lmax, H, d, -3, 3)
    q = torch.stack([q_all[b, n - 1] for b, n in enumerate(lens)]).contiguous()
    w = torch.stack([w_all[b, n - 1] for b, n in enumerate(lens)]).contiguous()
    pages = [(n + P - 1) // P for n in lens]
    num_pages = sum(pages) + 2
    perm = np.random.default_rng(3).permutation(num_pages)
    max_pages = max(pages)
    table = np.full((B, max_pages), -1, np.int32)
    pool = torch.zeros((num_pages * P, d), dtype=torch.bfloat16)
    nxt = 0
    for b, n in enumerate(lens):
        for lp in range(pages[b]):
            pp = int(perm[nxt])
            nxt += 1
            table[b, lp] = pp
            t0, t1 = lp * P, min(n, (lp + 1) * P)
            pool[pp * P:pp * P + t1 - t0] = k[b, t0:t1]
    ws = torch.zeros(dsa.idx_score_topk_paged_workspace_size(B, Lmax, H, d, topk), dtype=torch.uint8, device=DEV)
    idx = dsa.idx_score_topk_paged(q.to(DEV), pool.view(num_pages, P, d).to(DEV), torch.from_numpy(table).to(DEV),
                                   torch.tensor(lens, dtype=torch.int32, device=DEV), w.to(DEV), topk, Lmax,
                                   workspace=ws)
    assert dsa.read_status(ws) == 0
    idx = idx.cpu().numpy()
    for b, n in enumerate(lens):
        kl = oracle.gather_paged(pool.float().numpy(), table[b], n, P)
        sc = oracle.indexer_scores(q[b][None], kl, w[b][None], n - 1)
        _expect_identical(idx[b][None], oracle.topk_select(sc, topk, n - 1), f"paged b={b}")


def test_fused_selection_equals_oracle_selection_on_the_kernels_own_scores():
    """On ordinary (non-integer) inputs the fused kernel's selection is exactly the oracle's rule
    applied to the scores the same kernel exports (idx_scores shares its MMA and epilogue
    arithmetic): the streaming selection adds no error of its own."""
    B, L, H, d, topk = 1, 5000, 32, 128, 2048
    g = synth.StructuredIndexer("h32_5000", B, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    q, k, w = g.layer(0)
    qd, kd, wd = q.to(DEV), k.to(DEV), w.to(DEV)
    idx = dsa.idx_score_topk(qd, kd, wd, topk).cpu().numpy()[0]
    sc = dsa.idx_scores(qd, kd, wd).cpu().numpy()[0]
    _expect_identical(idx, oracle.topk_select(sc, topk), "fused vs own scores")
    # the standalone selection on the same score array is the same rule
    sel = dsa.idx_topk_scores(torch.from_numpy(sc).to(DEV), topk).cpu().numpy()
    _expect_identical(sel, oracle.topk_select(sc, topk), "idx_topk_scores")
