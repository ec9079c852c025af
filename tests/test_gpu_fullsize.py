"""Parity at the full workload sizes, in the launch configuration the bench times, on sampled
rows the oracle computes one by one: the 200K-token prefill group, the 16K-token prefill group
(64 indexer heads, 32/32 attention heads), the 64 x 200K decode step, the last chunk of the
1M-token chunked prefill and a decode step after it (fp8 indexer, latent attention)."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth
from dsa_checks import check_attention, check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"
H_I, D_I, TOPK, HQ, HKV, DH = 32, 128, 2048, 32, 4, 128


def test_prefill_200k_sampled_rows():
    L = 200000
    gen = synth.StructuredIndexer("fullsize_prefill", 1, L, H_I, D_I, r=32, base_std=1.0, noise_std=0.12,
                                  device=DEV, seed=11)
    q, k, w = gen.layer(0)
    del gen
    layers = []
    for l in range(2):
        Q, K, V = synth.attention_inputs("fullsize_prefill", l, 1, L, L, HQ, HKV, DH, DH, device=DEV, seed=11)
        lay = {"Q": Q, "K": K, "V": V, "O": torch.empty((1, L, HQ, DH), dtype=torch.bfloat16, device=DEV)}
        if l == 0:
            lay.update(q_I=q, k_I=k, w=w)
        layers.append(lay)
    shape = dsa.group_shape(1, L, 0, L, H_I, D_I, HQ, HKV, DH, DH, TOPK, o_dtype=dsa.DSA_BF16)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=DEV)
    cache = dsa.IndexCache(torch.empty((1, L, TOPK), dtype=torch.int32, device=DEV))
    dsa.layer_group_forward(shape, layers, "FS", cache, workspace=ws)
    assert dsa.read_status(ws) == 0
    rows = np.array([0, 2047, 2048, 99999, 150000, L - 1])
    idx = cache.buf[0, rows].cpu().numpy()
    kk = k[0].cpu()
    for j, t in enumerate(rows):
        sc = oracle.indexer_scores(q[0, t:t + 1].cpu(), kk[: t + 1], w[0, t:t + 1].cpu(), int(t))
        check_selection(idx[j:j + 1], oracle.topk_select(sc, TOPK, int(t)), sc, int(t), TOPK, rtol=1e-3)
    for lay in layers:
        O = lay["O"][0, rows].float().cpu().numpy()
        ref = oracle.sparse_attention(lay["Q"][0, rows].cpu(), lay["K"][0].cpu(), lay["V"][0].cpu(), idx)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
        assert np.all(np.abs(O - ref) <= 2e-3 + 0.5 * ulp)


def test_decode_64x200k_sampled_sequences():
    B, L = 64, 200000
    gen = synth.StructuredIndexer("fullsize_decode", B, L, H_I, D_I, r=32, base_std=1.0, noise_std=0.12,
                                  device=DEV, seed=12)
    q, w = gen.queries(0, L - 1, L)
    k = gen.keys(0)
    del gen
    Q, K, V = synth.attention_inputs("fullsize_decode", 0, B, 1, L, HQ, HKV, DH, DH, device=DEV, seed=12)
    idx = dsa.idx_score_topk(q, k, w, TOPK, q_pos0=L - 1)
    O = dsa.sparse_attn_topk(Q, K, V, idx)
    idx_h = idx.cpu().numpy()
    O = O.cpu().numpy()
    for b in (0, 31, 63):
        sc = oracle.indexer_scores(q[b].cpu(), k[b].cpu(), w[b].cpu(), L - 1)
        check_selection(idx_h[b], oracle.topk_select(sc, TOPK, L - 1), sc, L - 1, TOPK, rtol=1e-3)
        ref = oracle.sparse_attention(Q[b].cpu(), K[b].cpu(), V[b].cpu(), idx_h[b])
        check_attention(O[b], ref)


def test_1m_tail_chunk_sampled_rows():
    """Last 8192-token chunk of a 1048576-token prefill: fp8 indexer (H_I=64) and latent attention."""
    L1, C, H1, HQ1 = 1 << 20, 8192, 64, 64
    p0 = L1 - C
    gen = synth.StructuredIndexer("fullsize_1m", 1, L1, H1, D_I, r=32, base_std=1.0, noise_std=0.1, device=DEV,
                                  seed=13)
    q, w = gen.queries(0, p0, L1)
    k = gen.keys(0)
    del gen
    q8, qs = synth.quantize_e4m3_rows(q)
    k8, ks = synth.quantize_e4m3_rows(k)
    del q, k
    Q, KV, _ = synth.attention_inputs("fullsize_1m", 0, 1, C, L1, HQ1, 1, 576, None, device=DEV, seed=13)
    idx = dsa.idx_score_topk(q8, k8, w, TOPK, q_pos0=p0, q_scale=qs, k_scale=ks)
    O = dsa.sparse_attn_topk(Q, KV, None, idx, d_v=512)
    rows = np.array([0, C - 1])
    idx_h = idx[0, rows].cpu().numpy()
    k8h, ksh = k8[0].cpu().numpy(), ks[0].cpu().numpy()
    for j, i in enumerate(rows):
        t = p0 + int(i)
        sc = oracle.indexer_scores_fp8(q8[0, i:i + 1].cpu().numpy(), qs[0, i:i + 1].cpu().numpy(), k8h[: t + 1],
                                       ksh[: t + 1], w[0, i:i + 1].cpu(), t)
        check_selection(idx_h[j:j + 1], oracle.topk_select(sc, TOPK, t), sc, t, TOPK, rtol=2e-2)
    ref = oracle.sparse_attention(Q[0, rows].cpu(), KV[0].cpu(), None, idx_h, d_v=512)
    check_attention(O[0, rows].cpu().numpy(), ref)


def test_prefill_16k_group_sampled_rows():
    """The 16K-token prefill group FSSS (H_I=64, d_I=128 bf16, top-2048; attention 32 query and 32 KV
    heads, d=128) through layer_group_forward, checked on rows 0, k-1, k, the middle and the end."""
    L, H16, HQ16, HKV16 = 16384, 64, 32, 32
    gen = synth.StructuredIndexer("fullsize_16k", 1, L, H16, D_I, r=32, base_std=1.0, noise_std=0.2,
                                  device=DEV, seed=14)
    q, k, w = gen.layer(0)
    del gen
    layers = []
    for l in range(4):
        Q, K, V = synth.attention_inputs("fullsize_16k", l, 1, L, L, HQ16, HKV16, DH, DH, device=DEV, seed=14)
        lay = {"Q": Q, "K": K, "V": V, "O": torch.empty((1, L, HQ16, DH), dtype=torch.float32, device=DEV)}
        if l == 0:
            lay.update(q_I=q, k_I=k, w=w)
        layers.append(lay)
    shape = dsa.group_shape(1, L, 0, L, H16, D_I, HQ16, HKV16, DH, DH, TOPK)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=DEV)
    cache = dsa.IndexCache(torch.empty((1, L, TOPK), dtype=torch.int32, device=DEV))
    stats = dsa.layer_group_forward(shape, layers, "FSSS", cache, workspace=ws)
    assert dsa.read_status(ws) == 0
    assert stats.indexer_launches == 1 and stats.attention_launches == 4
    rows = np.array([0, TOPK - 1, TOPK, L // 2, L - 2, L - 1])
    idx = cache.buf[0, rows].cpu().numpy()
    kk = k[0].cpu()
    for j, t in enumerate(rows):
        sc = oracle.indexer_scores(q[0, t:t + 1].cpu(), kk[: t + 1], w[0, t:t + 1].cpu(), int(t))
        check_selection(idx[j:j + 1], oracle.topk_select(sc, TOPK, int(t)), sc, int(t), TOPK, rtol=1e-3)
    for lay in layers:
        ref = oracle.sparse_attention(lay["Q"][0, rows].cpu(), lay["K"][0].cpu(), lay["V"][0].cpu(), idx)
        check_attention(lay["O"][0, rows].cpu().numpy(), ref)


def test_decode_after_1m_prefill_fp8_latent():
    """The first decode step after the 1048576-token prefill (the new token is position 1048576, so the
    cache holds 1048577 tokens): the split fp8 decode indexer (H_I=64) and the split latent attention
    (64 heads) through layer_group_forward with the bench's pattern FSSSFSSS, in the bench's launch
    configuration; every layer checked."""
    n_kv, H1, HQ1 = (1 << 20) + 1, 64, 64
    gen = synth.StructuredIndexer("fullsize_dec1m", 1, n_kv, H1, D_I, r=32, base_std=1.0, noise_std=0.1,
                                  device=DEV, seed=15)
    q, w = gen.queries(0, n_kv - 1, n_kv)
    k = gen.keys(0)
    q8, qs = synth.quantize_e4m3_rows(q)
    k8, ks = synth.quantize_e4m3_rows(k)
    q2, w2 = gen.queries(4, n_kv - 1, n_kv)
    k2 = gen.keys(4)
    q82, qs2 = synth.quantize_e4m3_rows(q2)
    k82, ks2 = synth.quantize_e4m3_rows(k2)
    del gen, q, k, q2, k2
    pattern = "FSSSFSSS"
    layers = []
    for l in range(8):
        Q, KV, _ = synth.attention_inputs("fullsize_dec1m", l, 1, 1, n_kv, HQ1, 1, 576, None, device=DEV, seed=15)
        lay = {"Q": Q, "K": KV, "V": None, "O": torch.empty((1, 1, HQ1, 512), dtype=torch.float32, device=DEV)}
        if l == 0:
            lay.update(q_I=q8, q_scale=qs, k_I=k8, k_scale=ks, w=w)
        if l == 4:
            lay.update(q_I=q82, q_scale=qs2, k_I=k82, k_scale=ks2, w=w2)
        layers.append(lay)
    shape = dsa.group_shape(1, 1, n_kv - 1, n_kv, H1, D_I, HQ1, 1, 576, 512, TOPK, idx_dtype=dsa.DSA_E4M3)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=DEV)
    cache = dsa.IndexCache(torch.empty((1, 1, TOPK), dtype=torch.int32, device=DEV))
    # layers 0-3 (F layer 0's selection), checked before layers 4-7 overwrite the cache
    dsa.layer_group_forward(shape, layers[:4], pattern[:4], cache, workspace=ws)
    assert dsa.read_status(ws) == 0
    groups = [(0, cache.buf.cpu().numpy()[0].copy())]
    dsa.layer_group_forward(shape, layers[4:], pattern[4:], cache, workspace=ws)
    assert dsa.read_status(ws) == 0
    groups.append((4, cache.buf.cpu().numpy()[0].copy()))
    for f, idx in groups:
        L_ = layers[f]
        sc = oracle.indexer_scores_fp8(L_["q_I"][0].cpu().numpy(), L_["q_scale"][0].cpu().numpy(),
                                       L_["k_I"][0].cpu().numpy(), L_["k_scale"][0].cpu().numpy(),
                                       L_["w"][0].cpu(), n_kv - 1)
        check_selection(idx, oracle.topk_select(sc, TOPK, n_kv - 1), sc, n_kv - 1, TOPK, rtol=2e-2)
        sel = torch.from_numpy(idx[0]).long().to(DEV)
        for l in range(f, f + 4):
            # the oracle sees only the selected rows (renumbered 0..k-1; attention is order-free)
            rows_kv = layers[l]["K"][0, sel].cpu()
            ref = oracle.sparse_attention(layers[l]["Q"][0].cpu(), rows_kv, None,
                                          np.arange(TOPK, dtype=np.int32)[None], d_v=512)
            check_attention(layers[l]["O"][0].cpu().numpy(), ref)
