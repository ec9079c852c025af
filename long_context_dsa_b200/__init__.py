"""B200-native DSA indexer with cross-layer index reuse (IndexCache / IndexShare).

The compute path is the C-ABI library ``libdsa.so`` built from ``csrc/``
(hand-written CUDA for sm_100a).  ``long_context_dsa_b200.dsa`` is the thin
ctypes binding with the same entry-point names; it loads the library on
first use and raises if it is missing.  ``synth`` draws seeded inputs.
"""
