"""Context-parallel prefill, host side (CPU, gloo): the zig-zag row plan covers the
sequence once and balances the causal work, the key all-gather rebuilds the sequence
in order on every rank (2 and 3 ranks), and running each rank's blocks as chunks of
prefill over the gathered keys reproduces the single-sequence result (the oracle does
the arithmetic here; the GPU executor is checked in test_gpu_context_parallel)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_dsa_b200 import context_parallel as cp
from long_context_dsa_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("W", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("L", [1, 2, 127, 128, 129, 300, 1000, 4097, 200000])
def test_blocks_cover_the_sequence_once(L, W):
    owner = np.full(L, -1)
    for r in range(W):
        p = cp.make_plan(L, W, r)
        assert p.padded_len >= L and p.padded_len - L < 2 * W
        a = cp.make_plan(L, W, r, align=128)
        assert a.blk % 128 == 0 and a.padded_len >= L
        for s, e in p.blocks:
            assert 0 <= s <= e <= L
            assert np.all(owner[s:e] == -1), "row owned twice"
            owner[s:e] = r
    assert np.all(owner >= 0), "row owned by nobody"


def test_block_order_is_zigzag():
    W = 4
    plans = [cp.make_plan(8 * 1024, W, r) for r in range(W)]
    starts = [[s // 1024 for s, _ in p.blocks] for p in plans]
    assert starts == [[0, 7], [1, 6], [2, 5], [3, 4]]


@pytest.mark.parametrize("L,W,align", [(1, 1, 128), (300, 2, 128), (700, 3, 16), (1000, 4, 64), (4097, 3, 128)])
def test_work_counts_against_brute_force(L, W, align):
    topk = 100
    for r in range(W):
        p = cp.make_plan(L, W, r, align)
        rows = [t for s, e in p.blocks for t in range(s, e)]
        assert cp.indexer_work(p) == sum(t + 1 for t in rows)
        assert cp.attention_work(p, topk) == sum(min(topk, t + 1) for t in rows)
        assert p.n_rows == len(rows)


def test_zigzag_balances_the_causal_triangle():
    L, W, k = 200000, 8, 2048
    plans = [cp.make_plan(L, W, r) for r in range(W)]
    iw = [cp.indexer_work(p) for p in plans]
    aw = [cp.attention_work(p, k) for p in plans]
    assert sum(iw) == L * (L + 1) // 2
    assert max(iw) / min(iw) < 1.001
    assert len(set(iw[1:])) == 1            # ranks without the clipped last block cost the same
    # attention reads min(k, t+1) rows: only rank 0's first k rows are lighter, the rest are equal
    assert len(set(aw[1:])) == 1 and aw[0] < aw[1] and aw[1] / aw[0] < 1.05
    # a contiguous split of the same rows would leave the last rank (2W-1)x the first's indexer work
    per = -(-L // W)
    contiguous = [sum(t + 1 for t in range(r * per, min(L, (r + 1) * per))) for r in range(W)]
    assert max(contiguous) / min(contiguous) > 10


def test_local_rows_round_trip_and_one_rank_gather():
    L = 300
    x = torch.arange(L * 3, dtype=torch.float32).view(1, L, 3)
    p = cp.make_plan(L, 1, 0)
    loc = cp.local_rows(x, p)
    assert loc.shape == (2, p.blk, 3)
    g = cp.allgather_keys(loc, p)          # one rank: a view of the local buffer, no process group
    assert g.data_ptr() == loc.data_ptr()
    assert torch.equal(g[:, :L], x) and torch.all(g[:, L:] == 0)
    back = cp.scatter_rows(loc, p, torch.zeros_like(x))
    assert torch.equal(back, x)
    with pytest.raises(ValueError):
        cp.local_rows(x[:, :10], p)
    with pytest.raises(ValueError):
        cp.make_plan(L, 2, 2)


# ------------------------------------------------------------- gloo ranks
PATTERN = "FSFS"
SHAPE = dict(L=700, H=4, d=32, Hq=4, Hkv=2, dh=32, topk=32, align=16)


def _inputs():
    s = SHAPE
    g = synth.StructuredIndexer("cp", 1, s["L"], s["H"], s["d"], r=4, base_std=1.0, noise_std=0.2, seed=3)
    layers = []
    for l, kind in enumerate(PATTERN):
        Q, K, V = synth.attention_inputs("cp", l, 1, s["L"], s["L"], s["Hq"], s["Hkv"], s["dh"], s["dh"], seed=3)
        Lh = {"Q": Q, "K": K, "V": V}
        if kind == "F":
            Lh["q_I"], Lh["k_I"], Lh["w"] = g.layer(l)
        layers.append(Lh)
    return layers


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = SHAPE
        plan = cp.make_plan(s["L"], world, rank, s["align"])
        layers = _inputs()          # every rank draws the same sequence and keeps its own rows
        ok_gather = True
        res = []
        for Lh in layers:
            g = {}
            for name in ("k_I", "K", "V"):
                if name in Lh:
                    full = Lh[name].float()
                    got = cp.allgather_keys(cp.local_rows(full, plan), plan)
                    ok_gather &= bool(torch.equal(got[:, : s["L"]], full)) and bool(torch.all(got[:, s["L"]:] == 0))
                    # into a caller buffer, as the bench does every step (stale contents overwritten)
                    buf = torch.full((2 * world, plan.blk) + tuple(full.shape[2:]), 7.0)
                    got2 = cp.allgather_keys(cp.local_rows(full, plan), plan, out=buf)
                    ok_gather &= got2.data_ptr() == buf.data_ptr() and bool(torch.equal(got2, got))
                    g[name] = got
            res.append(g)
        # each block is a chunk of prefill over the gathered keys (oracle arithmetic)
        blocks = []
        for slot, (b0, b1) in enumerate(plan.blocks):
            if b1 <= b0:
                continue
            blk_layers = []
            for Lh, g in zip(layers, res):
                d = {"Q": cp.local_rows(Lh["Q"], plan)[slot, : b1 - b0],
                     "K": g["K"][0, :b1], "V": g["V"][0, :b1]}
                if "q_I" in Lh:
                    d["q_I"] = cp.local_rows(Lh["q_I"], plan)[slot, : b1 - b0]
                    d["w"] = cp.local_rows(Lh["w"], plan)[slot, : b1 - b0]
                    d["k_I"] = g["k_I"][0, :b1]
                blk_layers.append(d)
            idxs, outs, calls = oracle.layer_group_forward(blk_layers, PATTERN, s["topk"], q_pos0=b0)
            blocks.append((b0, b1, [np.asarray(i) for i in idxs], [np.asarray(o) for o in outs], calls))
        out[rank] = (ok_gather, blocks)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_reproduce_the_single_sequence(world):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    s = SHAPE
    layers = [{n: t[0] for n, t in Lh.items()} for Lh in _inputs()]
    ref_idx, ref_out, ref_calls = oracle.layer_group_forward(layers, PATTERN, s["topk"])
    covered = np.zeros(s["L"], dtype=bool)
    for r in range(world):
        ok_gather, blocks = res[r]
        assert ok_gather
        for b0, b1, idxs, outs, calls in blocks:
            assert calls == ref_calls                     # every block runs the F layers only
            covered[b0:b1] = True
            for l in range(len(PATTERN)):
                np.testing.assert_array_equal(idxs[l], np.asarray(ref_idx[l])[b0:b1])
                np.testing.assert_allclose(outs[l], np.asarray(ref_out[l])[b0:b1], rtol=0, atol=1e-12)
    assert covered.all()
