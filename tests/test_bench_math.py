"""The roofline arithmetic bench.py reports, checked on CPU against brute-force sums and the
closed forms of the workload (200K prefill, top-2048, H_I=32, d_I=128, GQA 32/4, d=128)."""

import importlib.util
import os

import pytest

from long_context_dsa_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)      # defines functions only; main() is not run
    return mod


@pytest.mark.parametrize("L,k", [(1, 1), (5, 3), (100, 100), (1000, 64), (4097, 2048)])
def test_gathered_rows_is_the_sum_of_min_k_t1(bench, L, k):
    assert bench.gathered_rows(L, k) == sum(min(k, t + 1) for t in range(L))


def test_workload_totals(bench):
    L, k = 200000, 2048
    # indexer: every causal (query, key) pair costs H_I * d_I multiply-adds
    assert bench.indexer_flops() == 2 * 32 * 128 * (L * (L + 1) // 2) == 163840819200000
    # attention: each gathered row is a K and a V slice of d bf16 values per KV head
    assert bench.attn_bytes() == bench.gathered_rows(L, k) * 4 * 2 * 128 * 2 == 834567929856
    # DRAM traffic of one full launch: the read and write bytes of one ncu capture, summed
    assert bench.attn_traffic() == round(22.01e9 + 1.64e9)


def test_step_roofline_matches_the_pages_configuration(bench):
    hbm, burst, sustained, _ = bench.peaks()
    t_idx = 2 * bench.indexer_flops() / (sustained * 1e12)     # two F layers per group
    t_gather = 8 * bench.attn_bytes() / (hbm * 1e9)           # eight attention layers
    assert t_gather > t_idx                                   # the gather bounds the step
    assert 0.9 < t_gather < 1.2                               # ~1.02 s at ~6.5 TB/s


def test_context_parallel_plan_of_the_workload():
    L = 200000
    for W in (2, 4, 8):
        plans = [cp.make_plan(L, W, r) for r in range(W)]
        assert sum(p.n_rows for p in plans) == L
        work = [cp.indexer_work(p) for p in plans]
        assert sum(work) == L * (L + 1) // 2
        assert max(work) / (sum(work) / W) < 1.001


def test_stratified_random_indices_are_causal_distinct_ascending(bench):
    import numpy as np
    idx = bench.stratified_random_indices(3000, 128, "cpu", 5, rows_per_chunk=1000)[0].numpy()
    for t in range(0, 3000, 7):
        n = min(128, t + 1)
        row = idx[t]
        assert np.all(row[n:] == -1)
        assert np.all(np.diff(row[:n]) > 0) and row[0] >= 0 and row[n - 1] <= t
        if t + 1 > 128:  # one token from each of the 128 strata of [0, t]
            strata = (np.arange(128) * (t + 1)) // 128
            assert np.all(row[:n] >= strata) and np.all(row[:n] < np.append(strata[1:], t + 1))
