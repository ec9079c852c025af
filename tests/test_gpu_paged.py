"""Paged, variable-length decode (idx_score_topk_paged, sparse_attn_topk_paged) against the
oracle on the logical caches the page tables describe."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth
from dsa_checks import check_attention, check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _paged_batch(name, lens, P, H, d, Hq, Hkv, dh, seed):
    B, Lmax = len(lens), max(lens)
    gen = synth.StructuredIndexer(name, B, Lmax, H, d, r=32, base_std=1.0, noise_std=0.2, seed=seed)
    k = gen.keys(0)                                           # [B, Lmax, d]
    q = torch.stack([gen.queries(0, n - 1, n)[0][b, 0] for b, n in enumerate(lens)])   # [B, H, d]
    w = torch.stack([gen.w[b, n - 1] for b, n in enumerate(lens)]).contiguous()        # [B, H]
    _, K, V = synth.attention_inputs(name, 0, B, 1, Lmax, Hq, Hkv, dh, dh, seed=seed)
    Q = synth.normal((B, Hq, dh), synth.seed_for(seed, name, "Qdec"), dtype=torch.bfloat16)
    pages = [(n + P - 1) // P for n in lens]
    num_pages = sum(pages) + 3
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)
    max_pages = max(pages) + 1
    table = np.full((B, max_pages), -1, np.int32)
    k_pool = torch.zeros((num_pages * P, d), dtype=torch.bfloat16)
    K_pool = torch.zeros((num_pages * P, Hkv, dh), dtype=torch.bfloat16)
    V_pool = torch.zeros((num_pages * P, Hkv, dh), dtype=torch.bfloat16)
    nxt = 0
    for b, n in enumerate(lens):
        for lp in range(pages[b]):
            pp = int(perm[nxt])
            nxt += 1
            table[b, lp] = pp
            t0, t1 = lp * P, min(n, (lp + 1) * P)
            k_pool[pp * P:pp * P + t1 - t0] = k[b, t0:t1]
            K_pool[pp * P:pp * P + t1 - t0] = K[b, t0:t1]
            V_pool[pp * P:pp * P + t1 - t0] = V[b, t0:t1]
    return dict(q=q, w=w, k_pool=k_pool, K_pool=K_pool, V_pool=V_pool, Q=Q, table=table,
                lens=np.array(lens, np.int32), num_pages=num_pages)


@pytest.mark.parametrize("P", [64, 256])
def test_paged_decode_matches_oracle(P):
    lens = [1, 100, 1500, 3000, 4097]
    H, d, k, Hq, Hkv, dh = 32, 128, 512, 32, 4, 128
    bt = _paged_batch(f"paged{P}", lens, P, H, d, Hq, Hkv, dh, 7)
    B = len(lens)
    table = torch.from_numpy(bt["table"]).to(DEV)
    seq = torch.from_numpy(bt["lens"]).to(DEV)
    k_pages = bt["k_pool"].view(bt["num_pages"], P, d).to(DEV)
    ws = torch.zeros(dsa.idx_score_topk_paged_workspace_size(B, max(lens), H, d, k), dtype=torch.uint8, device=DEV)
    idx = dsa.idx_score_topk_paged(bt["q"].to(DEV), k_pages, table, seq, bt["w"].to(DEV), k, max(lens),
                                   workspace=ws)
    assert dsa.read_status(ws) == 0
    idx_h = idx.cpu().numpy()
    for b, n in enumerate(lens):
        kl = oracle.gather_paged(bt["k_pool"].float().numpy(), bt["table"][b], n, P)
        ora = oracle.indexer_scores(bt["q"][b][None], kl, bt["w"][b][None], n - 1)
        ora_idx = oracle.topk_select(ora, k, n - 1)
        check_selection(idx_h[b][None], ora_idx, ora, n - 1, k, rtol=1e-3)

    Kp = bt["K_pool"].view(bt["num_pages"], P, Hkv, dh).to(DEV)
    Vp = bt["V_pool"].view(bt["num_pages"], P, Hkv, dh).to(DEV)
    wsa = torch.zeros(dsa.sparse_attn_topk_workspace_size(B, 1, bt["num_pages"] * P, Hq, Hkv, dh, dh, k),
                      dtype=torch.uint8, device=DEV)
    O = dsa.sparse_attn_topk_paged(bt["Q"].to(DEV), Kp, Vp, table, seq, idx, workspace=wsa)
    assert dsa.read_status(wsa) == 0
    O = O.cpu().numpy()
    for b, n in enumerate(lens):
        Kl = oracle.gather_paged(bt["K_pool"].float().numpy(), bt["table"][b], n, P)
        Vl = oracle.gather_paged(bt["V_pool"].float().numpy(), bt["table"][b], n, P)
        ref = oracle.sparse_attention(bt["Q"][b][None], Kl, Vl, idx_h[b][None])
        check_attention(O[b][None], ref)


def test_paged_decode_flags_bad_lengths_and_indices():
    lens = [300, 200]
    P, H, d, k, Hq, Hkv, dh = 64, 32, 128, 64, 8, 8, 64
    bt = _paged_batch("paged_bad", lens, P, H, d, Hq, Hkv, dh, 9)
    table = torch.from_numpy(bt["table"]).to(DEV)
    bad_len = torch.tensor([0, 200], dtype=torch.int32, device=DEV)
    k_pages = bt["k_pool"].view(bt["num_pages"], P, d).to(DEV)
    ws = torch.zeros(dsa.idx_score_topk_paged_workspace_size(2, 300, H, d, k), dtype=torch.uint8, device=DEV)
    dsa.idx_score_topk_paged(bt["q"].to(DEV), k_pages, table, bad_len, bt["w"].to(DEV), k, 300, workspace=ws)
    assert dsa.read_status(ws) & dsa.STATUS_BAD_INDEX
    # a length above max_seq_len (here still within the sequence's pages) is flagged and clamped
    # to max_seq_len: the per-sequence score slots hold max_seq_len keys
    assert bt["table"].shape[1] * P > 350
    ws.zero_()
    long_len = torch.tensor([350, 200], dtype=torch.int32, device=DEV)
    out = dsa.idx_score_topk_paged(bt["q"].to(DEV), k_pages, table, long_len, bt["w"].to(DEV), k, 300,
                                   workspace=ws)
    assert dsa.read_status(ws) & dsa.STATUS_BAD_INDEX
    assert int(out.max()) < 300
    # an index at or beyond its sequence's length is skipped and flagged
    seq = torch.from_numpy(bt["lens"]).to(DEV)
    idx = torch.full((2, k), -1, dtype=torch.int32)
    idx[0, :3] = torch.tensor([0, 5, 299])
    idx[1, :3] = torch.tensor([1, 2, 250])
    Kp = bt["K_pool"].view(bt["num_pages"], P, Hkv, dh).to(DEV)
    Vp = bt["V_pool"].view(bt["num_pages"], P, Hkv, dh).to(DEV)
    wsa = torch.zeros(dsa.sparse_attn_topk_workspace_size(2, 1, bt["num_pages"] * P, Hq, Hkv, dh, dh, k),
                      dtype=torch.uint8, device=DEV)
    O = dsa.sparse_attn_topk_paged(bt["Q"].to(DEV), Kp, Vp, table, seq, idx.to(DEV), workspace=wsa)
    assert dsa.read_status(wsa) & dsa.STATUS_BAD_INDEX
    Kl = oracle.gather_paged(bt["K_pool"].float().numpy(), bt["table"][1], 200, P)
    Vl = oracle.gather_paged(bt["V_pool"].float().numpy(), bt["table"][1], 200, P)
    ref = oracle.sparse_attention(bt["Q"][1][None], Kl, Vl, np.array([[1, 2, -1]]))
    check_attention(O.cpu().numpy()[1][None], ref)


def _random_selection(lens, k, seed):
    """Ascending distinct positions below each sequence's length, -1 padded (any valid selection)."""
    rng = np.random.default_rng(seed)
    idx = np.full((len(lens), k), -1, np.int32)
    for b, n in enumerate(lens):
        m = min(k, n)
        idx[b, :m] = np.sort(rng.choice(n, size=m, replace=False))
    return idx


def _fp8_pools(bt, P, Hkv, dh):
    K8, ks = synth.quantize_e4m3_rows(bt["K_pool"])    # [rows, Hkv, dh] codes, [rows, Hkv] scales
    V8, vs = synth.quantize_e4m3_rows(bt["V_pool"])
    n = bt["num_pages"]
    dev = (K8.view(n, P, Hkv, dh).to(DEV), ks.view(n, P, Hkv).to(DEV), V8.view(n, P, Hkv, dh).to(DEV),
           vs.view(n, P, Hkv).to(DEV))
    real = (oracle.dequantize_e4m3(K8.numpy(), ks.numpy()), oracle.dequantize_e4m3(V8.numpy(), vs.numpy()))
    return dev, real


def _fp8_tol(V_real):
    # each V element reaches the MMA as fp16(fp16(scale) * code): two roundings of 2^-11 relative;
    # an output row is a convex combination of V rows, so its error is at most that of one element.
    # Q is taken to fp16 (exact for these values) and P is split into fp16 hi + lo (~2^-22).
    return 2.5 * 2.0 ** -11 * float(np.abs(V_real).max()) + 2e-4


# (name, lens, P, Hq, Hkv, dh, k, o_dtype): few rows -> split ranges + merge; many rows -> one pass
FP8_CASES = [
    ("split_d128", [1, 100, 1500, 3000, 4097], 64, 32, 4, 128, 512, torch.float32),
    ("split_d64_bf16", [7, 64, 65, 2000], 16, 8, 8, 64, 256, torch.bfloat16),
    ("onepass_d128", list(np.random.default_rng(3).integers(20, 300, size=520)), 32, 8, 8, 128, 64, torch.float32),
]


@pytest.mark.parametrize("case", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_paged_fp8_kv_attention_matches_oracle(case):
    name, lens, P, Hq, Hkv, dh, k, o_dtype = case
    lens = [int(n) for n in lens]
    bt = _paged_batch("fp8" + name, lens, P, 32, 128, Hq, Hkv, dh, 11)
    B = len(lens)
    table = torch.from_numpy(bt["table"]).to(DEV)
    seq = torch.from_numpy(bt["lens"]).to(DEV)
    idx_h = _random_selection(lens, k, 12)
    (K8, ks, V8, vs), (K_real, V_real) = _fp8_pools(bt, P, Hkv, dh)
    wsa = torch.zeros(dsa.sparse_attn_topk_workspace_size(B, 1, bt["num_pages"] * P, Hq, Hkv, dh, dh, k),
                      dtype=torch.uint8, device=DEV)
    O = dsa.sparse_attn_topk_paged_e4m3(bt["Q"].to(DEV), K8, ks, V8, vs, table, seq, torch.from_numpy(idx_h).to(DEV),
                                        o_dtype=o_dtype, workspace=wsa)
    assert dsa.read_status(wsa) == 0
    O = O.float().cpu().numpy()
    tol = _fp8_tol(V_real) + (2.0 ** -9 * 4 if o_dtype == torch.bfloat16 else 0.0)   # bf16 output rounding
    for b, n in enumerate(lens):
        Kl = oracle.gather_paged(K_real, bt["table"][b], n, P)
        Vl = oracle.gather_paged(V_real, bt["table"][b], n, P)
        ref = oracle.sparse_attention(bt["Q"][b][None], Kl, Vl, idx_h[b][None])
        check_attention(O[b][None], ref, atol=tol)


def test_paged_fp8_kv_flags_bad_indices():
    lens = [300, 200]
    P, Hq, Hkv, dh, k = 64, 8, 8, 64, 64
    bt = _paged_batch("fp8_bad", lens, P, 32, 128, Hq, Hkv, dh, 9)
    table = torch.from_numpy(bt["table"]).to(DEV)
    seq = torch.from_numpy(bt["lens"]).to(DEV)
    idx = torch.full((2, k), -1, dtype=torch.int32)
    idx[0, :3] = torch.tensor([0, 5, 299])
    idx[1, :3] = torch.tensor([1, 2, 250])          # 250 >= 200: skipped and flagged
    (K8, ks, V8, vs), (K_real, V_real) = _fp8_pools(bt, P, Hkv, dh)
    wsa = torch.zeros(dsa.sparse_attn_topk_workspace_size(2, 1, bt["num_pages"] * P, Hq, Hkv, dh, dh, k),
                      dtype=torch.uint8, device=DEV)
    O = dsa.sparse_attn_topk_paged_e4m3(bt["Q"].to(DEV), K8, ks, V8, vs, table, seq, idx.to(DEV), workspace=wsa)
    assert dsa.read_status(wsa) & dsa.STATUS_BAD_INDEX
    Kl = oracle.gather_paged(K_real, bt["table"][1], 200, P)
    Vl = oracle.gather_paged(V_real, bt["table"][1], 200, P)
    ref = oracle.sparse_attention(bt["Q"][1][None], Kl, Vl, np.array([[1, 2, -1]]))
    check_attention(O.cpu().numpy()[1][None], ref, atol=_fp8_tol(V_real))
