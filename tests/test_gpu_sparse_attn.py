"""Sparse attention over selected tokens (sparse_attn_topk) against the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth
from dsa_checks import check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _indices(L, k, seed, q_pos0=0, n_q=None, B=1):
    """Causal top-k index rows from random scores (selection itself is not under test here)."""
    n_q = L - q_pos0 if n_q is None else n_q
    rng = np.random.default_rng(seed)
    out = []
    for b in range(B):
        sc = rng.standard_normal((n_q, L)).astype(np.float32)
        out.append(oracle.topk_select(sc, k, q_pos0))
    return np.stack(out)


# (name, B, n_q, q_pos0, n_kv, Hq, Hkv, d, k, sample_rows)
CASES = [
    ("tiny512_mha8_d64", 1, 512, 0, 512, 8, 8, 64, 64, None),
    ("mha32_d128", 1, 400, 0, 400, 32, 32, 128, 256, None),
    ("gqa32x4_d128_k2048", 1, 2300, 0, 2300, 32, 4, 128, 2048, 160),
    ("gqa16x2_d128", 1, 300, 0, 300, 16, 2, 128, 100, None),
    ("gqa8x1_d128", 1, 200, 0, 200, 8, 1, 128, 50, None),
    ("gqa4x4_d64", 1, 300, 0, 300, 4, 4, 64, 33, None),
    ("decode_b4", 4, 1, 4999, 5000, 32, 4, 128, 2048, None),
    ("decode_b64_d64", 64, 1, 2999, 3000, 16, 2, 64, 1000, None),
    ("decode_b16_mha8", 16, 1, 1999, 2000, 8, 8, 128, 2000, None),
    ("decode_b3_k37", 3, 1, 99, 100, 32, 4, 128, 37, None),
    ("chunk4_b8_k2048", 8, 4, 2996, 3000, 32, 4, 128, 2048, None),
    ("chunk_b2", 2, 100, 900, 1000, 32, 4, 128, 300, None),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_sparse_attention_matches_oracle(case):
    name, B, n_q, q_pos0, n_kv, Hq, Hkv, d, k, sample = case
    Q, K, V = synth.attention_inputs(name, 0, B, n_q, n_kv, Hq, Hkv, d, d)
    idx = _indices(n_kv, k, 1, q_pos0, n_q, B)
    ws = torch.zeros(dsa.sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d, d, k), dtype=torch.uint8,
                     device=DEV)
    O = dsa.sparse_attn_topk(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV), workspace=ws)
    assert dsa.read_status(ws) == 0
    O = O.cpu().numpy()
    rows = np.arange(n_q) if sample is None else np.unique(np.concatenate(
        [np.arange(8), np.arange(n_q - 8, n_q), np.random.default_rng(2).choice(n_q, sample, replace=False)]))
    for b in range(B):
        ref = oracle.sparse_attention(Q[b, rows], K[b], V[b], idx[b, rows])
        check_attention(O[b, rows], ref)


def test_dense_special_case_k_covers_context():
    """k >= L: every prior token is selected, so this is dense causal attention."""
    L, Hq, Hkv, d = 300, 8, 2, 128
    Q, K, V = synth.attention_inputs("dense", 0, 1, L, L, Hq, Hkv, d, d)
    idx = _indices(L, 512, 3)
    O = dsa.sparse_attn_topk(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV)).cpu()
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q[0].double().permute(1, 0, 2), K[0].double().repeat_interleave(G, 1).permute(1, 0, 2),
        V[0].double().repeat_interleave(G, 1).permute(1, 0, 2), is_causal=True).permute(1, 0, 2)
    check_attention(O[0].numpy(), ref.numpy())


def test_padding_anywhere_and_order_free():
    L, Hq, Hkv, d, k = 200, 32, 4, 128, 64
    Q, K, V = synth.attention_inputs("pad", 0, 1, L, L, Hq, Hkv, d, d)
    idx = _indices(L, k, 4)[0]
    rng = np.random.default_rng(5)
    mixed = np.full((L, k + 17), -1, np.int32)
    for t in range(L):
        v = idx[t][idx[t] >= 0]
        v = rng.permutation(v)
        pos = np.sort(rng.choice(k + 17, v.size, replace=False))
        mixed[t, pos] = v
    O = dsa.sparse_attn_topk(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(mixed[None]).to(DEV)).cpu().numpy()
    check_attention(O[0], oracle.sparse_attention(Q[0], K[0], V[0], idx))


def test_out_of_range_index_is_skipped_and_flagged():
    L, Hq, Hkv, d, k = 64, 8, 8, 64, 8
    Q, K, V = synth.attention_inputs("bad", 0, 1, L, L, Hq, Hkv, d, d)
    idx = _indices(L, k, 6)
    idx[0, 10, 0] = L + 5      # beyond the cache
    idx[0, 11, 1] = -7         # negative, not the -1 pad
    ws = torch.zeros(dsa.sparse_attn_topk_workspace_size(1, L, L, Hq, Hkv, d, d, k), dtype=torch.uint8, device=DEV)
    O = dsa.sparse_attn_topk(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV), workspace=ws)
    assert dsa.read_status(ws) & dsa.STATUS_BAD_INDEX
    clean = idx.copy()
    clean[0, 10, 0] = -1
    clean[0, 11, 1] = -1
    check_attention(O.cpu().numpy()[0], oracle.sparse_attention(Q[0], K[0], V[0], clean[0]))


def test_split_ranges_decode_flags_bad_index_and_merges():
    """Few rows -> the index list is cut into ranges merged afterwards; padding-only ranges stay neutral."""
    B, L, Hq, Hkv, d, k = 2, 3000, 32, 4, 128, 2048
    Q, K, V = synth.attention_inputs("split", 0, B, 1, L, Hq, Hkv, d, d)
    idx = _indices(L, k, 12, L - 1, 1, B)
    idx[0, 0, 700:1500] = -1     # whole ranges of padding in the middle
    idx[1, 0, 5] = L + 3
    need = dsa.sparse_attn_topk_workspace_size(B, 1, L, Hq, Hkv, d, d, k)
    assert need > 256            # split-range state is in use for this shape
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    O = dsa.sparse_attn_topk(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV), workspace=ws)
    assert dsa.read_status(ws) & dsa.STATUS_BAD_INDEX
    clean = idx.copy()
    clean[1, 0, 5] = -1
    O = O.cpu().numpy()
    for b in range(B):
        check_attention(O[b], oracle.sparse_attention(Q[b], K[b], V[b], clean[b]))


def test_bf16_output():
    L, Hq, Hkv, d, k = 500, 32, 4, 128, 128
    Q, K, V = synth.attention_inputs("bf16o", 0, 1, L, L, Hq, Hkv, d, d)
    idx = _indices(L, k, 7)
    O = dsa.sparse_attn_topk(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV),
                             o_dtype=torch.bfloat16).float().cpu().numpy()[0]
    ref = oracle.sparse_attention(Q[0], K[0], V[0], idx[0])
    # half a bf16 ulp of the reference on top of the fp32 bar
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(O - ref) <= 2e-3 + 0.5 * ulp)


# latent (MLA-style) form: one 576-dim row per token is the key, its first 512 dims the value
LATENT = [
    ("latent_h64", 1, 300, 0, 300, 64, 128, None),
    ("latent_h16_chunk_b2", 2, 100, 400, 500, 16, 300, None),
    ("latent_h8_k64", 1, 200, 0, 200, 8, 64, None),
    ("latent_h64_k2048", 1, 2600, 0, 2600, 64, 2048, 48),
    # one query row per sequence (decode): few (row, head block) units, so each unit's index list
    # is cut into ranges over the SMs and a second kernel merges them
    ("latent_decode_b1_h64", 1, 1, 4999, 5000, 64, 2048, None),
    ("latent_decode_b3_h16_k300", 3, 1, 999, 1000, 16, 300, None),
    ("latent_decode_b2_h8_k37", 2, 1, 199, 200, 8, 37, None),
    # rows shorter than k: most ranges hold only -1 entries and must drop out of the merge
    ("latent_decode_short_h64", 2, 1, 99, 100, 64, 2048, None),
]


@pytest.mark.parametrize("case", LATENT, ids=[c[0] for c in LATENT])
def test_latent_attention_matches_oracle(case):
    name, B, n_q, q_pos0, n_kv, Hq, k, sample = case
    Q, KV, _ = synth.attention_inputs(name, 0, B, n_q, n_kv, Hq, 1, 576, None)
    idx = _indices(n_kv, k, 8, q_pos0, n_q, B)
    ws = torch.zeros(dsa.sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, 1, 576, 512, k), dtype=torch.uint8,
                     device=DEV)
    O = dsa.sparse_attn_topk(Q.to(DEV), KV.to(DEV), None, torch.from_numpy(idx).to(DEV), d_v=512, workspace=ws)
    assert dsa.read_status(ws) == 0
    O = O.cpu().numpy()
    rows = np.arange(n_q) if sample is None else np.unique(np.concatenate(
        [np.arange(4), np.arange(n_q - 4, n_q), np.random.default_rng(9).choice(n_q, sample, replace=False)]))
    for b in range(B):
        ref = oracle.sparse_attention(Q[b, rows], KV[b], None, idx[b, rows], d_v=512)
        check_attention(O[b, rows], ref)


# several query tokens per sequence reuse one selection (multi-token decode)
# (name, B, n_q, q_pos0, n_kv, Hq, Hkv, d, k, q_per_idx)
SHARED = [
    ("mtp4_gqa", 3, 4, 2996, 3000, 32, 4, 128, 2048, 4),
    ("mtp_ragged_d64", 2, 5, 995, 1000, 16, 2, 64, 300, 2),
    ("mtp_b64", 64, 4, 1996, 2000, 32, 4, 128, 512, 4),
    ("mtp_latent", 2, 3, 497, 500, 16, 1, 576, 128, 3),
]


def _shared_rows(B, n_q, q_pos0, n_kv, k, q, seed):
    """Each group's selection is made for its last query (top-k of random scores up to that position)."""
    rng = np.random.default_rng(seed)
    n_rows = (n_q + q - 1) // q
    out = np.empty((B, n_rows, k), np.int32)
    for b in range(B):
        for r in range(n_rows):
            last = q_pos0 + min((r + 1) * q, n_q) - 1
            sc = rng.standard_normal((1, n_kv)).astype(np.float32)
            out[b, r] = oracle.topk_select(sc, k, last)[0]
    return out


@pytest.mark.parametrize("case", SHARED, ids=[c[0] for c in SHARED])
def test_shared_selection_matches_oracle(case):
    name, B, n_q, q_pos0, n_kv, Hq, Hkv, d, k, q = case
    latent = d == 576
    Q, K, V = synth.attention_inputs(name, 0, B, n_q, n_kv, Hq, Hkv, d, None if latent else d)
    idx = _shared_rows(B, n_q, q_pos0, n_kv, k, q, 21)
    d_v = 512 if latent else d
    ws = torch.zeros(dsa.sparse_attn_topk_workspace_size(B, n_q, n_kv, Hq, Hkv, d, d_v, k), dtype=torch.uint8,
                     device=DEV)
    O = dsa.sparse_attn_topk_shared(Q.to(DEV), K.to(DEV), None if latent else V.to(DEV),
                                    torch.from_numpy(idx).to(DEV), q, q_pos0, d_v=d_v, workspace=ws)
    assert dsa.read_status(ws) == 0
    O = O.cpu().numpy()
    for b in range(B):
        ref = oracle.sparse_attention_shared(Q[b], K[b], None if latent else V[b], idx[b], q, q_pos0,
                                             d_v=d_v if latent else None)
        check_attention(O[b], ref)


def test_shared_rejects_positions_outside_the_cache():
    Q, K, V = synth.attention_inputs("mtp_bad", 0, 1, 4, 100, 8, 8, 64, 64)
    idx = np.zeros((1, 1, 8), np.int32)
    with pytest.raises(dsa.DsaError):
        dsa.sparse_attn_topk_shared(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV), 4, 97)
