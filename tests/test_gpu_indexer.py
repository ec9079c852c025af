"""Fused indexer + top-k (idx_score_topk) and its scores (idx_scores) on the
GPU against the fp64 oracle, on seeded synthetic inputs spanning several
tiles with ragged tails."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth
from dsa_checks import check_scores, check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (name, B, n_q, q_pos0, n_kv, H, d, k, gen)
CASES = [
    # 512-token tiny group shape: H_I=4, d_I=64, top-64, rank-8 structure, noise N(0,1)/8
    ("tiny512", 1, 512, 0, 512, 4, 64, 64, dict(r=8, base_std=1 / 8, noise_std=1 / 8)),
    # 16K-prefill head shape (H_I=64, d_I=128) on 1200 tokens: 9.4 key tiles, ragged query tile
    ("h64_1200", 1, 1200, 0, 1200, 64, 128, 256, dict(r=32, base_std=1.0, noise_std=0.2)),
    # 200K-prefill head shape (H_I=32, d_I=128) with top-2048: rows below and above t = 2047,
    # candidate buffers pruned while streaming
    ("h32_5000", 1, 5000, 0, 5000, 32, 128, 2048, dict(r=32, base_std=1.0, noise_std=0.2)),
    # a later chunk of a chunked prefill, two sequences
    ("chunk_b2", 2, 300, 700, 1000, 64, 128, 128, dict(r=32, base_std=1.0, noise_std=0.2)),
    # decode: one query per sequence at the end of its cache
    ("decode_b3", 3, 1, 2999, 3000, 32, 128, 512, dict(r=32, base_std=1.0, noise_std=0.2)),
    ("h16_777", 1, 777, 0, 777, 16, 128, 100, dict(r=32, base_std=1.0, noise_std=0.2)),
    ("h8_640", 1, 640, 0, 640, 8, 128, 64, dict(r=32, base_std=1.0, noise_std=0.2)),
    # small top-k over many key tiles: frequent prunes, rows shorter than k at the start
    ("h32_k16", 1, 1500, 0, 1500, 32, 128, 16, dict(r=32, base_std=1.0, noise_std=0.2)),
    ("h64_k1", 1, 600, 0, 600, 64, 128, 1, dict(r=32, base_std=1.0, noise_std=0.2)),
    ("h4_k3_b2", 2, 700, 0, 700, 4, 64, 3, dict(r=8, base_std=1 / 8, noise_std=1 / 8)),
    # decode through the split kernel: long caches, one query per sequence, query inside the cache
    ("decode_b2_h64", 2, 1, 19999, 20000, 64, 128, 2048, dict(r=32, base_std=1.0, noise_std=0.2)),
    ("decode_mid_b4", 4, 1, 4000, 5000, 32, 128, 300, dict(r=32, base_std=1.0, noise_std=0.2)),
]


def _inputs(name, B, n_q, q_pos0, n_kv, H, d, gen):
    g = synth.StructuredIndexer(name, B, n_kv, H, d, seed=0, **gen)
    q, k, w = g.layer(0)
    q = q[:, q_pos0:q_pos0 + n_q].contiguous()
    w = w[:, q_pos0:q_pos0 + n_q].contiguous()
    return q, k, w


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_indexer_topk_matches_oracle(case):
    name, B, n_q, q_pos0, n_kv, H, d, k, gen = case
    q, kk, w = _inputs(name, B, n_q, q_pos0, n_kv, H, d, gen)
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, n_q, q_pos0, n_kv, H, d, k), dtype=torch.uint8, device=DEV)
    idx = dsa.idx_score_topk(q.to(DEV), kk.to(DEV), w.to(DEV), k, q_pos0=q_pos0, workspace=ws)
    assert dsa.read_status(ws) == 0
    scores = dsa.idx_scores(q.to(DEV), kk.to(DEV), w.to(DEV), q_pos0=q_pos0)
    idx = idx.cpu().numpy()
    scores = scores.cpu().numpy()
    for b in range(B):
        ora = oracle.indexer_scores(q[b], kk[b], w[b], q_pos0)
        check_scores(scores[b], ora, q_pos0, rtol=1e-3)
        ora_idx = oracle.topk_select(ora, k, q_pos0)
        frac = check_selection(idx[b], ora_idx, ora, q_pos0, k, rtol=1e-3)
        assert frac > 0.9, f"only {frac:.3f} of rows match exactly"


def test_indexer_fp8_matches_oracle():
    B, L, H, d, k = 1, 1500, 64, 128, 256
    g = synth.StructuredIndexer("fp8", B, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    q, kk, w = g.layer(0)
    q8, qs = synth.quantize_e4m3_rows(q)
    k8, ks = synth.quantize_e4m3_rows(kk)
    q8d, k8d = q8.to(DEV), k8.to(DEV)
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, L, 0, L, H, d, k, dsa.DSA_E4M3), dtype=torch.uint8,
                     device=DEV)
    idx = dsa.idx_score_topk(q8d, k8d, w.to(DEV), k, q_scale=qs.to(DEV), k_scale=ks.to(DEV), workspace=ws)
    assert dsa.read_status(ws) == 0
    scores = dsa.idx_scores(q8d, k8d, w.to(DEV), q_scale=qs.to(DEV), k_scale=ks.to(DEV)).cpu().numpy()
    ora = oracle.indexer_scores_fp8(q8[0].numpy(), qs[0].numpy(), k8[0].numpy(), ks[0].numpy(), w[0])
    # the arithmetic matches the dequantised oracle to fp32 accumulation error; 2e-2 is the fp8 bar
    check_scores(scores[0], ora, 0, rtol=2e-2)
    check_scores(scores[0], ora, 0, rtol=1e-3)
    frac = check_selection(idx.cpu().numpy()[0], oracle.topk_select(ora, k), ora, 0, k, rtol=2e-2)
    assert frac > 0.9
    # quantisation error against the bf16 originals (reported, not a parity gate)
    ora_bf = oracle.indexer_scores(q[0], kk[0], w[0])
    m = np.isfinite(ora_bf)
    rel = np.abs(ora[m] - ora_bf[m]) / np.maximum(np.abs(ora_bf[m]), 1e-2 * np.abs(ora_bf[m]).max())
    print(f"fp8 quantisation error vs bf16 originals: median {np.median(rel):.3e}, max {rel.max():.3e}")


def test_indexer_is_causal_under_perturbation():
    """Changing keys after position t never changes row t's selection."""
    B, L, H, d, k = 1, 700, 32, 128, 64
    q, kk, w = _inputs("causal", B, L, 0, L, H, d, dict(r=32, base_std=1.0, noise_std=0.2))
    a = dsa.idx_score_topk(q.to(DEV), kk.to(DEV), w.to(DEV), k).cpu()
    k2 = kk.clone()
    k2[:, 400:] = torch.randn_like(k2[:, 400:].float()).to(torch.bfloat16) * 4
    b = dsa.idx_score_topk(q.to(DEV), k2.to(DEV), w.to(DEV), k).cpu()
    assert torch.equal(a[:, :400], b[:, :400])


def test_indexer_repeatable():
    B, L, H, d, k = 1, 2100, 32, 128, 512
    q, kk, w = _inputs("rep", B, L, 0, L, H, d, dict(r=32, base_std=1.0, noise_std=0.2))
    qd, kd, wd = q.to(DEV), kk.to(DEV), w.to(DEV)
    a = dsa.idx_score_topk(qd, kd, wd, k)
    b = dsa.idx_score_topk(qd, kd, wd, k)
    assert torch.equal(a, b)


def test_indexer_survivors_concentrated_in_one_lane_range():
    """Keys whose position mod 128 is below 32 (one epilogue warp's lanes) score far above the
    rest, so one warp's candidate share holds most survivors and the prune must rebalance."""
    B, L, H, d, k = 1, 6000, 32, 128, 2048
    q, kk, w = _inputs("skew", B, L, 0, L, H, d, dict(r=32, base_std=1.0, noise_std=0.2))
    hot = (torch.arange(L) % 128) < 32
    kk = kk.float()
    kk[:, hot] *= 4.0  # a longer key scores higher through the ReLU in expectation
    kk = kk.to(torch.bfloat16)
    idx = dsa.idx_score_topk(q.to(DEV), kk.to(DEV), w.to(DEV), k).cpu().numpy()[0]
    ora = oracle.indexer_scores(q[0], kk[0], w[0])
    frac = check_selection(idx, oracle.topk_select(ora, k), ora, 0, k, rtol=1e-3)
    assert frac > 0.9


def test_decode_long_cache():
    """One query against a 1.7M-token cache (the score keys of the row, then the histogram-bin
    select); the selection follows the oracle's rule."""
    B, L, H, d, k = 1, 1_700_000, 32, 128, 2048
    g = synth.StructuredIndexer("long_decode", B, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    kk = g.keys(0)
    q, w = g.queries(0, L - 1, L)
    ws = torch.zeros(dsa.idx_score_topk_workspace_size(B, 1, L - 1, L, H, d, k), dtype=torch.uint8, device=DEV)
    idx = dsa.idx_score_topk(q.to(DEV), kk.to(DEV), w.to(DEV), k, q_pos0=L - 1, workspace=ws)
    assert dsa.read_status(ws) == 0
    ora = oracle.indexer_scores(q[0], kk[0], w[0], L - 1)
    ora_idx = oracle.topk_select(ora, k, L - 1)
    check_selection(idx.cpu().numpy()[0], ora_idx, ora, L - 1, k, rtol=1e-3)
