"""Comparison rules shared by the GPU parity tests.

Tolerances (floating point has no tolerance in the pages; these follow the
library's stated parity bar):
* scores: |g - o| <= rtol * max(|o|, 1e-2 * max_s |o[t, s]|), rtol 1e-3 for
  bf16 inputs and 2e-2 for e4m3 inputs.  The floor keeps near-zero ReLU sums
  from demanding a relative match.
* selection: the GPU and the oracle select the same number of indices per
  row; every index the GPU selects that the oracle did not must have an
  oracle score within that tolerance of the oracle's k-th score.
* attention: max |O_gpu - O_oracle| <= 2e-3 for fp32 output.
"""

import numpy as np


def score_tol(o_row, rtol):
    fin = o_row[np.isfinite(o_row)]
    floor = 1e-2 * (np.abs(fin).max() if fin.size else 0.0)
    return rtol * np.maximum(np.abs(o_row), floor)


def check_scores(gpu, ora, q_pos0, rtol):
    """gpu/ora: [n_q, n_kv]; compares the causal part of each row."""
    worst = 0.0
    for i in range(ora.shape[0]):
        n = q_pos0 + i + 1
        o = ora[i, :n].astype(np.float64)
        g = gpu[i, :n].astype(np.float64)
        tol = score_tol(o, rtol)
        err = np.abs(g - o)
        bad = np.nonzero(err > tol)[0]
        assert bad.size == 0, f"row {i}: {bad.size} scores off, e.g. s={bad[0]} gpu={g[bad[0]]} oracle={o[bad[0]]}"
        worst = max(worst, float((err / np.maximum(tol / rtol, 1e-30)).max()))
    return worst  # max relative error (in units of the floor-adjusted magnitude)


def check_selection(gpu_idx, ora_idx, ora_scores, q_pos0, k, rtol):
    """Rule: same count; each GPU-only index scores within tolerance of the oracle's k-th score.
    Also checks canonical layout (ascending, then -1) and causality.  Returns the exact-match fraction."""
    n_q = gpu_idx.shape[0]
    exact = 0
    for i in range(n_q):
        p = q_pos0 + i
        g = gpu_idx[i]
        o = ora_idx[i]
        cnt = min(k, p + 1)
        gv = g[:cnt]
        assert np.all(g[cnt:] == -1), f"row {i}: padding"
        assert np.all(gv >= 0) and np.all(gv <= p), f"row {i}: non-causal or missing index"
        assert np.all(np.diff(gv) > 0), f"row {i}: not strictly ascending"
        if np.array_equal(g, o):
            exact += 1
            continue
        row = ora_scores[i, :p + 1].astype(np.float64)
        kth = np.sort(row)[::-1][cnt - 1]
        tol = score_tol(row, rtol)
        tk = rtol * max(abs(kth), 1e-2 * np.abs(row).max())
        extra = np.setdiff1d(gv, o[:cnt])
        assert np.all(row[extra] >= kth - tk), (
            f"row {i}: GPU picked index scoring {row[extra].min()} < k-th {kth} - {tk}")
        del tol
    return exact / max(n_q, 1)


def check_attention(gpu, ora, atol=2e-3):
    err = np.abs(gpu.astype(np.float64) - ora)
    m = float(err.max()) if err.size else 0.0
    assert m <= atol, f"max abs error {m} > {atol}"
    return m
