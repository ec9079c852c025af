"""Top-k selection on the GPU (idx_topk_scores) against the oracle, bit for bit,
on identical fp32 score arrays."""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run(scores_np, k, q_pos0):
    s = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).to(DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    out = dsa.idx_topk_scores(s, k, q_pos0=q_pos0, workspace=ws)
    bits = dsa.read_status(ws)
    return out.cpu().numpy(), bits


def test_ties_fixture_bit_exact():
    cases = json.load(open(os.path.join(GOLDEN, "topk_ties.json")))["cases"]
    for c in cases:
        row = np.array([float(v) if isinstance(v, str) else v for v in c["row"]], np.float32)
        got, bits = _run(row[None, :], c["k"], q_pos0=row.size - 1)
        assert bits == 0
        assert got[0].tolist() == c["expect"], c


@pytest.mark.parametrize("k", [1, 7, 64, 300, 1024, 2048])
def test_random_with_many_ties(k):
    rng = np.random.default_rng(k)
    rows, n_kv, q_pos0 = 300, 4000, 3700
    sc = (rng.integers(-40, 40, size=(rows, n_kv)) * 0.25).astype(np.float32)
    sc[rng.random(sc.shape) < 0.1] = np.float32(-0.0)
    sc[rng.random(sc.shape) < 0.05] = np.float32(0.0)
    got, bits = _run(sc, k, q_pos0)
    assert bits == 0
    exp = oracle.topk_select(sc, k, q_pos0)
    assert np.array_equal(got, exp)


def test_all_equal_and_short_rows():
    rows, n_kv = 64, 64
    sc = np.zeros((rows, n_kv), np.float32)
    for k in (1, 5, 63, 64, 100):
        got, bits = _run(sc, k, 0)
        assert bits == 0 and np.array_equal(got, oracle.topk_select(sc, k, 0))


def test_streaming_prunes_long_rows():
    """Rows far longer than the candidate buffer, ascending scores (every key enters, many prunes)."""
    n_kv, rows = 60000, 6
    base = np.arange(n_kv, dtype=np.float32) * np.float32(1e-3)
    sc = np.stack([base, base[::-1].copy(), np.sin(np.arange(n_kv)).astype(np.float32),
                   np.zeros(n_kv, np.float32), np.round(np.cos(np.arange(n_kv) * 0.01) * 8).astype(np.float32),
                   np.random.default_rng(1).standard_normal(n_kv).astype(np.float32)])
    for k in (2048, 777):
        got, bits = _run(sc, k, n_kv - rows)
        assert bits == 0
        assert np.array_equal(got, oracle.topk_select(sc, k, n_kv - rows))


def test_indexer_shaped_scores_c2_rows():
    """Scores of the 16K prefill shape (H_I=64, d_I=128) from the oracle, two row blocks."""
    L, H, d, k = 16384, 64, 128, 2048
    g = synth.StructuredIndexer("c2", 1, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    q, kk, w = g.layer(0)
    for p0, n in ((L - 48, 48), (2000, 96)):
        sc = oracle.indexer_scores(q[0, p0:p0 + n], kk[0], w[0, p0:p0 + n], q_pos0=p0)
        got, bits = _run(sc, k, p0)
        assert bits == 0
        assert np.array_equal(got, oracle.topk_select(sc, k, p0))


def test_nan_is_flagged():
    sc = np.zeros((4, 16), np.float32)
    sc[2, 3] = np.nan
    _, bits = _run(sc, 2, 12)
    assert bits & dsa.STATUS_NAN_SCORE


def test_survivors_concentrated_in_one_warp():
    """High scores only where (position mod 128) < 32: one warp's share of the candidate buffer
    fills with survivors, forcing the ordered rebalance inside the prune."""
    n_kv, rows = 30000, 4
    rng = np.random.default_rng(21)
    sc = rng.standard_normal((rows, n_kv)).astype(np.float32)
    hot = (np.arange(n_kv) % 128) < 32
    sc[:, hot] += 10.0
    for k in (2048, 1500):
        got, bits = _run(sc, k, n_kv - rows)
        assert bits == 0
        assert np.array_equal(got, oracle.topk_select(sc, k, n_kv - rows))
