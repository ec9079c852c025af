"""Host side of the F/S pattern search in libdsa (greedy over an overlap matrix) against the
oracle's greedy, and its argument checks.  No GPU needed: the search runs on the host."""

import numpy as np
import pytest

import oracle
from long_context_dsa_b200 import dsa


@pytest.mark.parametrize("seed", range(12))
def test_library_search_equals_oracle(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 13))
    # dyadic values: every loss is exact in double, so both sides break ties the same way
    ov = rng.integers(0, 65, size=(n, n)) / 64.0
    for n_f in range(1, n + 1):
        assert dsa.layer_pattern_search(ov, n_f) == oracle.pattern_search(ov, n_f)


def test_library_search_block_structure():
    blocks = [0, 0, 0, 1, 1, 1, 2, 2]
    ov = np.array([[0.9 if a == b else 0.3 for b in blocks] for a in blocks])
    assert dsa.layer_pattern_search(ov, 3) == "FSSFSSFS"


def test_library_search_rejects_bad_arguments():
    ov = np.full((4, 4), 0.5)
    for n_f in (0, 5):
        with pytest.raises(dsa.DsaError):
            dsa.layer_pattern_search(ov, n_f)
    bad = ov.copy()
    bad[1, 3] = 1.5
    with pytest.raises(dsa.DsaError):
        dsa.layer_pattern_search(bad, 2)
