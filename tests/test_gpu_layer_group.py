"""layer_group_forward: F layers index, S layers reuse the cache byte for byte
and launch no indexer work; every layer attends with its own Q/K/V."""

import numpy as np
import pytest
import torch

import oracle
from long_context_dsa_b200 import dsa, synth
from dsa_checks import check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("pattern", ["FSSS", "FSSSFSSS", "FFFF"])
def test_layer_group_against_oracle(pattern):
    """The whole group against the oracle's own group composition (its selections, its cache,
    its attention).  The indexer inputs are integers with quarter-step weights, so every score
    is exact in fp32 and the GPU's selections must equal the oracle's byte for byte; every
    layer's output, in every group of the pattern, is then checked against the oracle's."""
    B, L, H, d, Hq, Hkv, dh, k = 1, 512, 4, 64, 8, 8, 64, 64
    layers = []
    for l in range(len(pattern)):
        Q, K, V = synth.attention_inputs("grp" + pattern, l, B, L, L, Hq, Hkv, dh, dh)
        Lh = {"Q": Q, "K": K, "V": V}
        if pattern[l] == "F":
            Lh["q_I"], Lh["k_I"], Lh["w"] = synth.integer_indexer(f"grp{pattern}/{l}", B, L, H, d, -4, 4)
        layers.append(Lh)
    dev_layers = []
    for Lh in layers:
        dl = {n: t.to(DEV) for n, t in Lh.items()}
        dl["O"] = torch.empty((B, L, Hq, dh), dtype=torch.float32, device=DEV)
        dev_layers.append(dl)
    cache = dsa.IndexCache(torch.full((B, L, k), -7, dtype=torch.int32, device=DEV))
    shape = dsa.group_shape(B, L, 0, L, H, d, Hq, Hkv, dh, dh, k)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=DEV)
    stats = dsa.layer_group_forward(shape, dev_layers, pattern, cache, workspace=ws)
    dsa.check_status(ws)
    assert stats.indexer_launches == pattern.count("F")
    assert stats.attention_launches == len(pattern)
    ora_idx, ora_out, calls = oracle.layer_group_forward([{n: t[0] for n, t in Lh.items()} for Lh in layers],
                                                         pattern, k)
    assert calls == pattern.count("F")
    # the cache ends with the last F layer's selection, byte for byte the oracle's
    assert np.array_equal(cache.buf.cpu().numpy()[0], ora_idx[-1])
    for l in range(len(pattern)):
        check_attention(dev_layers[l]["O"].cpu().numpy()[0], ora_out[l])


def test_s_layers_get_the_same_buffer():
    B, L, H, d, k = 1, 256, 4, 64, 32
    cache = dsa.IndexCache(torch.zeros((B, L, k), dtype=torch.int32, device=DEV))
    cache.put(0, "FSSS")
    for l in range(4):
        t = dsa.idx_cache_get(cache, l, "FSSS")
        assert t.data_ptr() == cache.buf.data_ptr()
    with pytest.raises(dsa.DsaError):
        dsa.idx_cache_get(cache, 4, "FSSSFSSS")


def test_fsss_runs_a_quarter_of_the_indexer_work():
    """Indexer time of FSSS x2 vs all-F on the 200K head shape at reduced length: >= 3x less.
    The library records an event before and after each layer's indexer launch (none on S
    layers); the indexer time is the sum of those intervals, measured on the launch stream."""
    B, L, H, d, Hq, Hkv, dh, k = 1, 8192, 32, 128, 32, 4, 128, 2048
    g = synth.StructuredIndexer("ratio", B, L, H, d, r=32, base_std=1.0, noise_std=0.2, device=DEV, seed=0)
    layers = []
    for l in range(8):
        Q, K, V = synth.attention_inputs("ratio", l, B, L, L, Hq, Hkv, dh, dh, device=DEV)
        q, kk, w = g.layer(l)
        layers.append({"Q": Q, "K": K, "V": V, "q_I": q, "k_I": kk, "w": w,
                       "O": torch.empty((B, L, Hq, dh), dtype=torch.float32, device=DEV)})
    shape = dsa.group_shape(B, L, 0, L, H, d, Hq, Hkv, dh, dh, k)
    ws = torch.zeros(dsa.layer_group_forward_workspace_size(shape), dtype=torch.uint8, device=DEV)
    cache = dsa.IndexCache(torch.empty((B, L, k), dtype=torch.int32, device=DEV))
    idx_ms = {}
    for pat in ("FFFFFFFF", "FSSSFSSS"):
        events = [torch.cuda.Event(enable_timing=True) for _ in range(3 * 8)]
        for e in events:
            e.record()
        for rep in range(3):  # the last repetition is measured
            stats = dsa.layer_group_forward(shape, layers, pat, cache, workspace=ws, events=events)
            torch.cuda.synchronize()
            assert stats.indexer_launches == pat.count("F")
        idx_ms[pat] = sum(events[3 * l].elapsed_time(events[3 * l + 1]) for l in range(8))
    dsa.check_status(ws)
    print(f"indexer ms: {idx_ms}")
    assert idx_ms["FFFFFFFF"] >= 3.0 * idx_ms["FSSSFSSS"]
