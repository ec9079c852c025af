"""F/S pattern search end to end on the GPU: every layer of a segmented synthetic group
runs as F, idx_overlap counts the shared selections (exactly the oracle's counts on the same
indices), and the greedy search keeps the indexer at the segment starts."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_pattern_search_on_segmented_group():
    n_layers, L, H, d, k = 8, 1200, 32, 128, 64
    gen = synth.SegmentedIndexer("pattern", 1, L, H, d, r=32, base_std=1.0, noise_std=0.2,
                                 segment_starts=[0, 3, 6], device=DEV, seed=5)
    idx = []
    for l in range(n_layers):
        q, kk, w = gen.layer(l)
        idx.append(dsa.idx_score_topk(q, kk, w, k))
    rows = torch.arange(L, device=DEV)
    counted = (rows + 1 > k)  # rows with more than k candidates (shorter rows select everything)
    ov = np.zeros((n_layers, n_layers))
    for f in range(n_layers):
        for j in range(f + 1, n_layers):
            c = dsa.idx_overlap(idx[f], idx[j])
            host = c.cpu().numpy()
            ref = oracle.overlap_counts(idx[f][0].cpu().numpy(), idx[j][0].cpu().numpy())
            assert np.array_equal(host, ref)
            ov[f, j] = float(c[counted].double().mean().item()) / k
    inside = [ov[f, j] for f in range(n_layers) for j in range(f + 1, n_layers) if gen.segment(f) == gen.segment(j)]
    across = [ov[f, j] for f in range(n_layers) for j in range(f + 1, n_layers) if gen.segment(f) != gen.segment(j)]
    assert min(inside) > 0.6 and max(across) < 0.3
    pattern = dsa.layer_pattern_search(ov, 3)
    assert pattern == "FSSFSSFS"
    assert pattern == oracle.pattern_search(ov, 3)
