"""Pins for the CPU oracle: checks against things other than itself.

Closed forms, hand-derived fixtures (tests/golden/), brute force by a
different route, library routines for special cases, and invariants.
Each group names the mistake it is there to catch.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import (IndexCache, check_pattern, e4m3_decode, indexer_scores,
                    indexer_scores_fp8, layer_group_forward, sparse_attention, sparse_attention_shared,
                    topk_overlap, topk_select)
from long_context_dsa_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(v):
    if isinstance(v, str):
        return float(v)  # "-0", "-1.4e-45"
    return v


# --------------------------------------------------------------------------
# indexer scores
# --------------------------------------------------------------------------

def test_scores_hand_worked_fixture():
    g = _fixture("indexer_tiny.json")
    sc = indexer_scores(np.array(g["q"], float), np.array(g["k"], float), np.array(g["w"], float))
    exp = np.array([[np.inf * -1 if v is None else v for v in row] for row in g["scores"]], np.float32)
    assert np.array_equal(sc, exp)
    for kk, rows in g["topk"].items():
        assert topk_select(sc, int(kk)).tolist() == rows


def test_scores_exact_rational_brute_force():
    """Small integer inputs: the exact score by rational arithmetic, one key at a time."""
    rng = np.random.default_rng(1)
    n, H, d = 9, 3, 5
    q = rng.integers(-4, 5, size=(n, H, d))
    k = rng.integers(-4, 5, size=(n, d))
    w = rng.integers(0, 7, size=(n, H)) / 4.0  # exact dyadic weights, H != n
    sc = indexer_scores(q.astype(float), k.astype(float), w)
    for t in range(n):
        for s in range(n):
            if s > t:
                assert sc[t, s] == -np.inf
                continue
            exact = Fraction(0)
            for h in range(H):
                dot = sum(int(q[t, h, j]) * int(k[s, j]) for j in range(d))
                if dot > 0:
                    exact += Fraction(w[t, h]) * dot
            assert sc[t, s] == np.float32(float(exact))


def test_scores_relu_drops_negative_heads():
    """All dot products negative -> every score is exactly zero (a dropped ReLU fails)."""
    q = -np.abs(np.random.default_rng(2).standard_normal((6, 4, 8))) - 0.1
    k = np.abs(np.random.default_rng(3).standard_normal((6, 8))) + 0.1
    w = np.ones((6, 4))
    sc = indexer_scores(q, k, w)
    assert np.all(sc[np.tril_indices(6)] == 0.0)


def test_scores_positive_inputs_closed_form():
    """q, k > 0 makes ReLU the identity: score = (sum_h w_h q_h) . k (another order of operations)."""
    rng = np.random.default_rng(4)
    n, H, d = 7, 5, 6
    q = rng.uniform(0.1, 1, (n, H, d))
    k = rng.uniform(0.1, 1, (n, d))
    w = rng.uniform(0, 1, (n, H))
    closed = np.einsum("th,thd->td", w, q) @ k.T
    sc = indexer_scores(q, k, w)
    m = np.tril(np.ones((n, n), bool))
    assert np.allclose(sc[m], closed[m].astype(np.float32), rtol=1e-6)


def test_scores_one_hot_weight_isolates_head():
    """w = e_h gives ReLU(q_h . k): catches a transposed w or head index."""
    rng = np.random.default_rng(5)
    n, H, d = 6, 3, 4
    q = rng.standard_normal((n, H, d))
    k = rng.standard_normal((n, d))
    for h in range(H):
        w = np.zeros((n, H))
        w[:, h] = 1.0
        sc = indexer_scores(q, k, w)
        ref = torch.relu(torch.from_numpy(q[:, h, :]) @ torch.from_numpy(k).T).numpy()
        m = np.tril(np.ones((n, n), bool))
        assert np.allclose(sc[m], ref[m].astype(np.float32), rtol=1e-6, atol=0)


def test_scores_causality_perturbation():
    """Changing k_I[s] for s > t leaves row t unchanged; row t includes s = t."""
    rng = np.random.default_rng(6)
    n, H, d = 10, 2, 4
    q = rng.standard_normal((n, H, d))
    k = rng.standard_normal((n, d))
    w = rng.uniform(0, 1, (n, H))
    base = indexer_scores(q, k, w)
    for t in range(n):
        k2 = k.copy()
        k2[t + 1:] = rng.standard_normal((n - t - 1, d)) * 50
        assert np.array_equal(indexer_scores(q, k2, w)[t], base[t])
    assert np.all(np.isfinite(np.diag(base)))


def test_scores_q_pos0_offset_equals_slice():
    """A chunk of queries at offset p0 scores exactly like those rows of the full problem."""
    rng = np.random.default_rng(7)
    n, H, d, p0 = 12, 2, 4, 5
    q = rng.standard_normal((n, H, d))
    k = rng.standard_normal((n, d))
    w = rng.uniform(0, 1, (n, H))
    full = indexer_scores(q, k, w)
    part = indexer_scores(q[p0:p0 + 4], k, w[p0:p0 + 4], q_pos0=p0)
    assert np.array_equal(part, full[p0:p0 + 4])


# --------------------------------------------------------------------------
# fp8 e4m3
# --------------------------------------------------------------------------

def test_e4m3_decode_all_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], lib[~nan])


def test_e4m3_known_code_points():
    v = e4m3_decode(np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0x40, 0x7E, 0xFE], np.uint8))
    assert v.tolist() == [0.0, -0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 2.0, 448.0, -448.0]


def test_fp8_scores_closed_form():
    """Codes for 1.0 / 2.0 / -1.0 with power-of-two scales: exact integer scores."""
    one, two, mone = 0x38, 0x40, 0xB8
    q8 = np.array([[[one, two]], [[mone, one]]], np.uint8)       # [2, H=1, d=2]
    k8 = np.array([[one, one], [two, mone]], np.uint8)            # [2, d=2]
    qs = np.array([[0.5], [4.0]], np.float32)
    ks = np.array([2.0, 0.25], np.float32)
    w = np.array([[1.0], [0.5]])
    sc = indexer_scores_fp8(q8, qs, k8, ks, w)
    # t=0,s=0: q=(0.5,1) k=(2,2) -> 3;  t=1,s=0: q=(-4,4) k=(2,2) -> 0 -> 0
    # t=1,s=1: q=(-4,4) k=(0.5,-0.25) -> -3 -> ReLU 0
    assert sc[0, 0] == 3.0 and sc[1, 0] == 0.0 and sc[1, 1] == 0.0


def test_fp8_power_of_two_rescale_changes_only_scale():
    """Doubling a key row keeps its codes, doubles its scale, doubles its scores."""
    x = synth.normal((6, 16), 11)
    x2 = x.clone()
    x2[3] *= 2
    c1, s1 = synth.quantize_e4m3_rows(x)
    c2, s2 = synth.quantize_e4m3_rows(x2)
    assert torch.equal(c1, c2) and s2[3] == 2 * s1[3]
    q = synth.normal((6, 2, 16), 12)
    qc, qs = synth.quantize_e4m3_rows(q)
    w = np.ones((6, 2))
    a = indexer_scores_fp8(qc.numpy(), qs.numpy(), c1.numpy(), s1.numpy(), w)
    b = indexer_scores_fp8(qc.numpy(), qs.numpy(), c2.numpy(), s2.numpy(), w)
    assert np.array_equal(b[3:, 3], 2 * a[3:, 3])
    others = [c for c in range(6) if c != 3]
    assert np.array_equal(a[:, others], b[:, others])


def test_dequantize_e4m3_code_points_and_scales():
    """Code x its row's scale, from the format: 0x38 = 1, 0x7E = 448, 0xB8 = -1, 0x01 = 2^-9."""
    codes = np.array([[0x38, 0x7E], [0xB8, 0x01]], np.uint8)
    v = oracle.dequantize_e4m3(codes, np.array([0.5, 3.0], np.float32))
    assert v.tolist() == [[0.5, 224.0], [-3.0, 3 * 2.0 ** -9]]
    # unit scales reduce to the plain decode; the scale of one row touches that row only
    c = np.arange(256, dtype=np.uint8).reshape(16, 16)
    ones = oracle.dequantize_e4m3(c, np.ones(16))
    assert np.array_equal(ones, e4m3_decode(c), equal_nan=True)
    sc = np.ones(16)
    sc[5] = 0.25
    v2 = oracle.dequantize_e4m3(c, sc)
    assert np.array_equal(v2[5], e4m3_decode(c[5]) * 0.25, equal_nan=True)
    assert np.array_equal(np.delete(v2, 5, 0), np.delete(ones, 5, 0), equal_nan=True)


def test_fp8_kv_cache_scales_act_on_scores_and_values():
    """Attention over a dequantized fp8 cache: a power-of-two K scale on every row equals that
    factor on Q; a V scale on every row scales the output by it."""
    rng = np.random.default_rng(5)
    Q = rng.standard_normal((1, 4, 16))
    K8 = synth.quantize_e4m3_rows(synth.normal((40, 2, 16), 21))[0].numpy()
    V8 = synth.quantize_e4m3_rows(synth.normal((40, 2, 16), 22))[0].numpy()
    ks = np.full((40, 2), 0.01)
    vs = np.full((40, 2), 0.02)
    idx = np.array([[0, 3, 17, 39, -1]])
    base = sparse_attention(Q, oracle.dequantize_e4m3(K8, ks), oracle.dequantize_e4m3(V8, vs), idx)
    k4 = sparse_attention(Q, oracle.dequantize_e4m3(K8, 4 * ks), oracle.dequantize_e4m3(V8, vs), idx)
    q4 = sparse_attention(4 * Q, oracle.dequantize_e4m3(K8, ks), oracle.dequantize_e4m3(V8, vs), idx)
    v3 = sparse_attention(Q, oracle.dequantize_e4m3(K8, ks), oracle.dequantize_e4m3(V8, 3 * vs), idx)
    np.testing.assert_allclose(k4, q4, rtol=1e-13, atol=0)
    np.testing.assert_allclose(v3, 3 * base, rtol=1e-13, atol=0)
    assert not np.allclose(k4, base)


# --------------------------------------------------------------------------
# top-k
# --------------------------------------------------------------------------

def _brute_rank_topk(row, k):
    """Select s iff fewer than k tokens beat it (pairwise count; a different algorithm)."""
    n = len(row)
    sel = []
    for s in range(n):
        better = sum(1 for u in range(n) if row[u] > row[s] or (row[u] == row[s] and u < s))
        if better < k:
            sel.append(s)
    return sel


def test_topk_ties_fixture():
    for case in _fixture("topk_ties.json")["cases"]:
        row = np.array([_num(v) for v in case["row"]], np.float32)
        n = row.size
        got = topk_select(row[None, :], case["k"], q_pos0=n - 1)[0].tolist()
        assert got == case["expect"], case


def test_topk_brute_force_pairwise_rank():
    rng = np.random.default_rng(8)
    for trial in range(40):
        n = int(rng.integers(1, 40))
        k = int(rng.integers(1, 12))
        # few distinct values -> many ties
        row = rng.integers(-3, 4, n).astype(np.float32) * np.float32(0.5)
        row[rng.random(n) < 0.2] = np.float32(-0.0)
        got = topk_select(row[None, :], k, q_pos0=n - 1)[0]
        exp = _brute_rank_topk(row.tolist(), k)
        assert got[:len(exp)].tolist() == exp and np.all(got[len(exp):] == -1)


def test_topk_short_rows_select_everything():
    sc = np.random.default_rng(9).standard_normal((8, 8)).astype(np.float32)
    out = topk_select(sc, k=8)
    for t in range(8):
        assert out[t, :t + 1].tolist() == list(range(t + 1))
        assert np.all(out[t, t + 1:] == -1)


def test_topk_causal_and_sorted():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((40, 2, 4))
    k = rng.standard_normal((40, 4))
    w = rng.uniform(0, 1, (40, 2))
    out = topk_select(indexer_scores(q, k, w), 6)
    for t in range(40):
        v = out[t][out[t] >= 0]
        assert v.size == min(6, t + 1) and np.all(v <= t) and np.all(np.diff(v) > 0)


# --------------------------------------------------------------------------
# sparse attention
# --------------------------------------------------------------------------

def _dense_causal_textbook(Q, K, V, scale):
    """Masked full-matrix softmax attention, written from the textbook definition."""
    n, Hq, _ = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.zeros((n, Hq, V.shape[2]))
    for h in range(Hq):
        S = Q[:, h, :] @ K[:, h // G, :].T * scale
        S[np.triu(np.ones((n, n), bool), 1)] = -np.inf
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        out[:, h, :] = P @ V[:, h // G, :]
    return out


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 1)])
def test_attention_dense_special_case(Hq, Hkv):
    """k >= L selects every prior token, so sparse attention is dense causal attention."""
    rng = np.random.default_rng(11)
    n, d, dv = 17, 8, 6
    Q = rng.standard_normal((n, Hq, d))
    K = rng.standard_normal((n, Hkv, d))
    V = rng.standard_normal((n, Hkv, dv))
    idx = topk_select(rng.standard_normal((n, n)).astype(np.float32), k=n + 3)
    got = sparse_attention(Q, K, V, idx)
    ref = _dense_causal_textbook(Q, K, V, 1 / math.sqrt(d))
    assert np.allclose(got, ref, atol=1e-12)
    # library routine: torch SDPA (fp64 CPU) with KV heads expanded for the group map
    G = Hq // Hkv
    Kx = torch.from_numpy(K).repeat_interleave(G, dim=1).permute(1, 0, 2)
    Vx = torch.from_numpy(V).repeat_interleave(G, dim=1).permute(1, 0, 2)
    lib = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q).permute(1, 0, 2), Kx, Vx, is_causal=True).permute(1, 0, 2).numpy()
    assert np.allclose(got, lib, atol=1e-12)


def test_attention_zero_query_is_mean_of_selected_values():
    rng = np.random.default_rng(12)
    n, k = 20, 5
    Q = np.zeros((n, 2, 4))
    K = rng.standard_normal((n, 1, 4))
    V = rng.standard_normal((n, 1, 3))
    idx = topk_select(rng.standard_normal((n, n)).astype(np.float32), k)
    out = sparse_attention(Q, K, V, idx)
    for t in range(n):
        sel = idx[t][idx[t] >= 0]
        assert np.allclose(out[t, 0], V[sel, 0].mean(axis=0), atol=1e-14)
        assert np.allclose(out[t, 1], out[t, 0], atol=0)


def test_attention_single_selected_token_returns_its_value():
    rng = np.random.default_rng(13)
    Q = rng.standard_normal((3, 2, 4)) * 10
    K = rng.standard_normal((5, 2, 4))
    V = rng.standard_normal((5, 2, 3))
    idx = np.array([[2, -1], [-1, 4], [0, -1]])
    out = sparse_attention(Q, K, V, idx)
    assert np.array_equal(out[0], V[2]) and np.array_equal(out[1], V[4]) and np.array_equal(out[2], V[0])


def test_attention_latent_form_equals_explicit_value_slice():
    rng = np.random.default_rng(14)
    n, Hq, dqk, dv = 9, 4, 12, 8
    Q = rng.standard_normal((n, Hq, dqk))
    lat = rng.standard_normal((n, 1, dqk))
    idx = topk_select(rng.standard_normal((n, n)).astype(np.float32), 4)
    a = sparse_attention(Q, lat, None, idx, d_v=dv)
    b = sparse_attention(Q, lat, lat[:, :, :dv].copy(), idx)
    assert np.array_equal(a, b)


def test_attention_invariant_to_order_and_padding_of_indices():
    rng = np.random.default_rng(15)
    n = 12
    Q = rng.standard_normal((n, 2, 4))
    K = rng.standard_normal((n, 2, 4))
    V = rng.standard_normal((n, 2, 4))
    idx = topk_select(rng.standard_normal((n, n)).astype(np.float32), 4)
    shuffled = np.full((n, 7), -1)
    for t in range(n):
        v = idx[t][idx[t] >= 0][::-1]
        pos = rng.choice(7, v.size, replace=False)
        shuffled[t, np.sort(pos)] = v
    assert np.allclose(sparse_attention(Q, K, V, idx), sparse_attention(Q, K, V, shuffled), atol=1e-14)


def test_shared_selection_with_one_query_per_row_is_plain_attention():
    rng = np.random.default_rng(16)
    n, p0 = 10, 20
    Q = rng.standard_normal((n, 4, 8))
    K = rng.standard_normal((p0 + n, 2, 8))
    V = rng.standard_normal((p0 + n, 2, 8))
    idx = topk_select(rng.standard_normal((n, p0 + n)).astype(np.float32), 6, p0)
    assert np.array_equal(sparse_attention_shared(Q, K, V, idx, 1, p0), sparse_attention(Q, K, V, idx))


def test_shared_selection_of_every_token_is_dense_causal_attention():
    """One shared row listing the whole prefix: each query of the group attends densely and
    causally up to its own position (torch SDPA with an explicit mask, fp64)."""
    rng = np.random.default_rng(17)
    n, p0, Hq, Hkv, d = 5, 11, 4, 2, 8
    Q = rng.standard_normal((n, Hq, d))
    K = rng.standard_normal((p0 + n, Hkv, d))
    V = rng.standard_normal((p0 + n, Hkv, d))
    row = np.arange(p0 + n)[None, :]
    got = sparse_attention_shared(Q, K, V, row, n, p0)
    G = Hq // Hkv
    mask = torch.from_numpy(np.arange(p0 + n)[None, :] <= (p0 + np.arange(n))[:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q).permute(1, 0, 2), torch.from_numpy(K).repeat_interleave(G, 1).permute(1, 0, 2),
        torch.from_numpy(V).repeat_interleave(G, 1).permute(1, 0, 2), attn_mask=mask).permute(1, 0, 2).numpy()
    assert np.allclose(got, ref, atol=1e-12)


def test_shared_selection_drops_entries_after_each_querys_position():
    rng = np.random.default_rng(18)
    n, p0 = 3, 6
    Q = rng.standard_normal((n, 2, 4))
    K = rng.standard_normal((p0 + n, 1, 4))
    V = rng.standard_normal((p0 + n, 1, 4))
    row = np.array([[1, 4, p0 + 1, p0 + 2, -1]])     # made for the group's last query
    got = sparse_attention_shared(Q, K, V, row, n, p0)
    assert np.array_equal(got[0], sparse_attention(Q[:1], K, V, np.array([[1, 4]]))[0])
    assert np.array_equal(got[1], sparse_attention(Q[1:2], K, V, np.array([[1, 4, p0 + 1]]))[0])
    assert np.array_equal(got[2], sparse_attention(Q[2:], K, V, np.array([[1, 4, p0 + 1, p0 + 2]]))[0])
    # ragged groups: q_per_idx = 2 over 3 queries uses rows 0, 0, 1
    rows2 = np.array([[0, 2, -1], [3, 5, p0 + 2]])
    got2 = sparse_attention_shared(Q, K, V, rows2, 2, p0)
    assert np.array_equal(got2[1], sparse_attention(Q[1:2], K, V, rows2[:1])[0])
    assert np.array_equal(got2[2], sparse_attention(Q[2:], K, V, rows2[1:])[0])


# --------------------------------------------------------------------------
# pattern, cache, layer group, chunking, overlap
# --------------------------------------------------------------------------

def test_overlap_counts_fixture():
    a = np.array([[0, 3, 5, 9, -1], [1, 2, 3, 4, 5], [-1, -1, -1, -1, -1]])
    b = np.array([[3, 4, 9, -1, -1], [0, 6, 7, 8, 9], [-1, -1, -1, -1, -1]])
    assert list(oracle.overlap_counts(a, b)) == [2, 0, 0]


def test_pattern_search_hand_worked_four_layers():
    """All-F loss 0.  One removal: layer 1 costs 0.1, layer 2 costs 1-0.6 = 0.4 (it reuses layer 1),
    layer 3 costs 0.05 -> FFFS.  Second removal: layer 1 gives 0.1 + 0.05 = 0.15, layer 2 gives
    (1-0.6) + (1-0.5) = 0.9 -> FSFS.  Third: FSSS."""
    ov = np.zeros((4, 4))
    ov[0, 1], ov[0, 2], ov[1, 2], ov[0, 3], ov[1, 3], ov[2, 3] = 0.9, 0.5, 0.6, 0.4, 0.5, 0.95
    assert oracle.pattern_search(ov, 4) == "FFFF"
    assert oracle.pattern_search(ov, 3) == "FFFS"
    assert oracle.pattern_search(ov, 2) == "FSFS"
    assert oracle.pattern_search(ov, 1) == "FSSS"
    assert oracle.pattern_loss(ov, "FSFS") == pytest.approx(0.15)


def test_pattern_search_finds_segment_starts_and_the_optimum():
    """Layers in blocks (0.9 inside a block, 0.3 across): with one F per block the greedy
    keeps exactly the block starts, which brute force over all patterns confirms is optimal."""
    import itertools
    blocks = [0, 0, 0, 1, 1, 1, 2, 2]
    n = len(blocks)
    ov = np.array([[0.9 if blocks[i] == blocks[j] else 0.3 for j in range(n)] for i in range(n)])
    got = oracle.pattern_search(ov, 3)
    assert got == "FSSFSSFS"
    best = min(("F" + "".join("F" if i + 1 in c else "S" for i in range(n - 1))
                for c in itertools.combinations(range(1, n), 2)), key=lambda p: oracle.pattern_loss(ov, p))
    assert oracle.pattern_loss(ov, got) == pytest.approx(oracle.pattern_loss(ov, best))


def test_gather_paged_identity_and_scatter_round_trip():
    rng = np.random.default_rng(19)
    P, n = 4, 10
    seq = rng.standard_normal((n, 3))
    # identity table over a pool that is the sequence itself (padded to whole pages)
    pool = np.concatenate([seq, np.zeros((2, 3))])
    assert np.array_equal(oracle.gather_paged(pool, [0, 1, 2], n, P), seq)
    # scattered into shuffled pages of a larger pool, gathered back
    perm = [5, 2, 7]
    big = np.full((8 * P, 3), np.nan)
    for lp, pp in enumerate(perm):
        chunk = seq[lp * P:(lp + 1) * P]
        big[pp * P:pp * P + len(chunk)] = chunk
    assert np.array_equal(oracle.gather_paged(big, perm + [-1, -1], n, P), seq)


@pytest.mark.parametrize("bad", ["", "S", "SFFF", "FXS", "fsss"])
def test_pattern_rejects(bad):
    with pytest.raises(ValueError):
        check_pattern(bad)


def test_cache_reuse_is_byte_identical_and_launch_free():
    rng = np.random.default_rng(16)
    n, H, d, Hq = 24, 2, 8, 2
    layers = []
    for l in range(8):
        L = {"Q": rng.standard_normal((n, Hq, d)), "K": rng.standard_normal((n, 1, d)),
             "V": rng.standard_normal((n, 1, d))}
        L["q_I"] = rng.standard_normal((n, H, d))
        L["k_I"] = rng.standard_normal((n, d))
        L["w"] = rng.uniform(0, 1, (n, H))
        layers.append(L)
    idxs, outs, calls = layer_group_forward(layers, "FSSSFSSS", topk=5)
    assert calls == 2
    for l in (1, 2, 3):
        assert idxs[l] is idxs[0]
    for l in (5, 6, 7):
        assert idxs[l] is idxs[4]
    assert not np.array_equal(idxs[0], idxs[4])
    # each S layer still attends with its own Q/K/V
    assert not np.allclose(outs[0], outs[1])
    assert np.array_equal(outs[2], sparse_attention(layers[2]["Q"], layers[2]["K"], layers[2]["V"], idxs[0]))
    # all-F computes every layer's own selection
    idx_f, _, calls_f = layer_group_forward(layers, "FFFFFFFF", topk=5)
    assert calls_f == 8 and np.array_equal(idx_f[4], idxs[4])


def test_cache_get_errors():
    c = IndexCache()
    with pytest.raises(ValueError):
        c.get(0, "F")
    c.put(0, np.zeros((1, 1)))
    with pytest.raises(ValueError):
        c.get(2, "FSF")  # layer 2 is F and has not written


def test_chunked_equals_unchunked():
    rng = np.random.default_rng(17)
    n, H, d, C, k = 32, 2, 4, 8, 5
    q = rng.standard_normal((n, H, d))
    kk = rng.standard_normal((n, d))
    w = rng.uniform(0, 1, (n, H))
    full = topk_select(indexer_scores(q, kk, w), k)
    parts = [topk_select(indexer_scores(q[c:c + C], kk[:c + C], w[c:c + C], q_pos0=c), k, q_pos0=c)
             for c in range(0, n, C)]
    assert np.array_equal(np.concatenate(parts), full)
    Q = rng.standard_normal((n, 2, 4))
    K = rng.standard_normal((n, 1, 4))
    V = rng.standard_normal((n, 1, 4))
    a = sparse_attention(Q, K, V, full)
    b = np.concatenate([sparse_attention(Q[c:c + C], K[:c + C], V[:c + C], full[c:c + C]) for c in range(0, n, C)])
    assert np.array_equal(a, b)


def test_decode_row_equals_last_prefill_row():
    rng = np.random.default_rng(18)
    n, H, d, k = 30, 3, 4, 6
    q = rng.standard_normal((n, H, d))
    kk = rng.standard_normal((n, d))
    w = rng.uniform(0, 1, (n, H))
    full = topk_select(indexer_scores(q, kk, w), k)
    dec = topk_select(indexer_scores(q[-1:], kk, w[-1:], q_pos0=n - 1), k, q_pos0=n - 1)
    assert np.array_equal(dec[0], full[-1])


def test_overlap_metric_closed_form():
    a = np.array([[0, 1, 2, 3], [4, 5, 6, 7]])
    b = np.array([[0, 1, 8, 9], [4, 5, 6, 9]])
    assert topk_overlap(a, b, 4, q_pos0=10) == pytest.approx((2 / 4 + 3 / 4) / 2)
    assert topk_overlap(a, a, 4, q_pos0=10) == 1.0


def test_structured_generator_overlap_in_reported_band():
    """Adjacent layers drawn by the structured recipe overlap 70-100% (the pages' band)."""
    L, H, d, k = 2048, 32, 128, 256
    g = synth.StructuredIndexer("pin", 1, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    rows = slice(L // 2, L)
    idx = []
    for l in range(2):
        q, kk, w = g.layer(l)
        sc = indexer_scores(q[0, rows], kk[0], w[0, rows], q_pos0=L // 2)
        idx.append(topk_select(sc, k, q_pos0=L // 2))
    ov = topk_overlap(idx[0], idx[1], k, q_pos0=L // 2)
    assert 0.70 <= ov <= 1.0, ov


def test_integer_generator_scores_are_exact_integers_over_four():
    """The exact-selection GPU tests rely on integer q/k and quarter-step w giving scores
    that fp32 holds exactly: check the oracle's rounded fp32 scores against int64 arithmetic
    (4 * score = sum_h (4 w) * max(0, q.k)), no floating point involved on that side."""
    q, k, w = synth.integer_indexer("pin_exact", 1, 64, 8, 128, -4, 4)
    qi = q[0].to(torch.int64).numpy()
    ki = k[0].to(torch.int64).numpy()
    w4 = (w[0] * 4).to(torch.int64).numpy()
    sc = indexer_scores(q[0], k[0], w[0])
    for t in range(64):
        dots = np.einsum("hd,sd->hs", qi[t], ki[:t + 1])
        exact = (w4[t][:, None] * np.maximum(dots, 0)).sum(axis=0)
        assert np.array_equal(sc[t, :t + 1].astype(np.float64) * 4, exact.astype(np.float64)), t
    # fp8 form: codes are small integers, scales powers of two, so the same holds in units of 2^-8
    q8, qs, k8, ks, w = synth.integer_indexer_e4m3("pin_exact8", 1, 48, 4, 128, -3, 3)
    assert set(np.unique(e4m3_decode(q8.numpy()))) <= set(range(-3, 4))
    sc8 = indexer_scores_fp8(q8[0].numpy(), qs[0].numpy(), k8[0].numpy(), ks[0].numpy(), w[0])
    qv = e4m3_decode(q8[0].numpy()).astype(np.int64)
    kv = e4m3_decode(k8[0].numpy()).astype(np.int64)
    qsi = np.rint(qs[0].numpy() * 8).astype(np.int64)   # q_scale in units of 2^-3
    ksi = np.rint(ks[0].numpy() * 8).astype(np.int64)
    w4 = np.rint(w[0].numpy() * 4).astype(np.int64)
    for t in range(48):
        dots = np.einsum("hd,sd->hs", qv[t], kv[:t + 1])
        exact = ksi[:t + 1] * (w4[t][:, None] * qsi[t][:, None] * np.maximum(dots, 0)).sum(axis=0)
        assert np.array_equal(sc8[t, :t + 1].astype(np.float64) * 4 * 64, exact.astype(np.float64)), t
