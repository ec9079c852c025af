"""Plain CPU oracle for the DSA indexer / IndexCache hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
and its Python binding) may import, call or link anything under
``oracle/``.  The only permitted users are ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``.

The oracle is numpy in float64.  It shares no code, headers, tables or
constants with the CUDA library; the two meet only in the seeded input
generator (``long_context_dsa_b200/synth.py``), which holds none of the
method's arithmetic.
"""

from .dsa_oracle import (  # noqa: F401
    e4m3_decode,
    dequantize_e4m3,
    indexer_scores,
    indexer_scores_fp8,
    topk_select,
    IndexCache,
    sparse_attention,
    sparse_attention_shared,
    layer_group_forward,
    topk_overlap,
    check_pattern,
    overlap_counts,
    pattern_loss,
    pattern_search,
    gather_paged,
)
