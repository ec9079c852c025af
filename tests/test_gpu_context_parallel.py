"""Context-parallel prefill on the GPU: each rank's blocks run through the library as
chunks of prefill over the gathered keys.  The ranks are emulated one after another on
one GPU (their kernels never wait on one another; the all-gather is replaced by the
sequence itself, whose order the gloo test checks).  The assembled selection of every
row is checked against the oracle, the outputs against the oracle's attention over that
selection, and both against the single-call layer group."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import context_parallel as cp
from long_context_dsa_b200 import dsa, synth
from dsa_checks import check_attention, check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layers(name, pattern, L, H, d, Hq, Hkv, dh):
    g = synth.StructuredIndexer(name, 1, L, H, d, r=32, base_std=1.0, noise_std=0.2, seed=0)
    layers = []
    for l, kind in enumerate(pattern):
        Q, K, V = synth.attention_inputs(name, l, 1, L, L, Hq, Hkv, dh, dh)
        Lh = {"Q": Q, "K": K, "V": V}
        if kind == "F":
            Lh["q_I"], Lh["k_I"], Lh["w"] = g.layer(l)
        layers.append(Lh)
    return layers


def _padded(x, n):
    out = torch.zeros((1, n) + tuple(x.shape[2:]), dtype=x.dtype, device=DEV)
    out[:, : x.shape[1]] = x.to(DEV)
    return out


# (name, L, world, pattern, H_I, d_I, topk, Hq, Hkv, d)
CASES = [
    ("cp2_3000", 3000, 2, "FSSS", 32, 128, 256, 8, 2, 128),
    ("cp3_2500", 2500, 3, "FSFS", 64, 128, 512, 8, 2, 64),
    # rank 0's second block lies past the end (L < 4 blocks of 128 with align=128)
    ("cp2_300_empty", 300, 2, "FS", 32, 128, 64, 4, 4, 128),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_context_parallel_matches_oracle_and_single_call(case):
    name, L, W, pattern, H, d, k, Hq, Hkv, dh = case
    align = 128 if name.endswith("empty") else 1
    layers = _layers(name, pattern, L, H, d, Hq, Hkv, dh)
    plans = [cp.make_plan(L, W, r, align) for r in range(W)]
    Lp = plans[0].padded_len
    # keys as every rank holds them after the all-gather
    keys = [{n: _padded(Lh[n], Lp) for n in ("k_I", "K", "V") if n in Lh} for Lh in layers]
    O = [torch.zeros((1, L, Hq, dh), dtype=torch.float32, device=DEV) for _ in layers]
    last_f = max(i for i, c in enumerate(pattern) if c == "F")
    idx_all = np.full((L, k), -7, dtype=np.int32)
    launches = 0
    for plan in plans:
        loc = []
        for Lh, kk in zip(layers, keys):
            d_ = {n: cp.local_rows(Lh[n].to(DEV), plan) for n in ("q_I", "w", "Q") if n in Lh}
            d_["O"] = torch.zeros((2, plan.blk, Hq, dh), dtype=torch.float32, device=DEV)
            d_.update(kk)
            loc.append(d_)
        ws = torch.zeros(cp.workspace_size(plan, H, d, Hq, Hkv, dh, dh, k), dtype=torch.uint8, device=DEV)
        cache_buf = torch.full((2, plan.blk, k), -7, dtype=torch.int32, device=DEV)
        n_idx, n_attn = cp.layer_group_forward(plan, loc, pattern, cache_buf, ws, H, d, Hq, Hkv, dh, dh, k)
        blocks = sum(1 for s, e in plan.blocks if e > s)
        assert n_idx == blocks * pattern.count("F") and n_attn == blocks * len(pattern)
        launches += n_idx + n_attn
        for slot, (s, e) in enumerate(plan.blocks):
            idx_all[s:e] = cache_buf[slot, : e - s].cpu().numpy()
        dsa.check_status(ws)
        for l in range(len(pattern)):
            cp.scatter_rows(loc[l]["O"], plan, O[l])
    # selection of the last F layer: every row against the oracle
    Lh = layers[last_f]
    ora = oracle.indexer_scores(Lh["q_I"][0], Lh["k_I"][0], Lh["w"][0])
    check_selection(idx_all, oracle.topk_select(ora, k), ora, 0, k, rtol=1e-3)
    # outputs of the layers that used it: the oracle's attention over the assembled selection
    for l in range(last_f, len(pattern)):
        ref = oracle.sparse_attention(layers[l]["Q"][0], layers[l]["K"][0], layers[l]["V"][0], idx_all)
        check_attention(O[l].cpu().numpy()[0], ref)
    # and the single-call layer group gives the same selection and (to rounding) the same outputs
    full = []
    for Lh in layers:
        d_ = {n: t.to(DEV) for n, t in Lh.items()}
        d_["O"] = torch.empty((1, L, Hq, dh), dtype=torch.float32, device=DEV)
        full.append(d_)
    cache = dsa.IndexCache(torch.empty((1, L, k), dtype=torch.int32, device=DEV))
    dsa.layer_group_forward(dsa.group_shape(1, L, 0, L, H, d, Hq, Hkv, dh, dh, k), full, pattern, cache)
    np.testing.assert_array_equal(cache.buf[0].cpu().numpy(), idx_all)
    for l in range(len(pattern)):
        torch.testing.assert_close(O[l], full[l]["O"], rtol=1e-4, atol=1e-5)
    assert launches == sum(1 for p in plans for s, e in p.blocks if e > s) * (pattern.count("F") + len(pattern))
