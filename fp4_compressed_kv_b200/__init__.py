"""B200-native compressed-KV sparse decode: FP4 (E2M1) 2:1-compressed KV
cache, int8 lightweight indexer with exact top-K, sparse attention over the
selected entries plus a sliding window, and CSA2 Full / Reindex / Reuse
layer groups.

The compute path is the C-ABI library ``libkvc.so`` built from ``csrc/``
(hand-written CUDA for sm_100a).  ``fp4_compressed_kv_b200.kvc`` is the thin
Python binding over it; ``fp4_compressed_kv_b200.synth`` holds the seeded
synthetic workloads.  Importing this package loads nothing: the binding
loads the library on first use and raises if it is missing.
"""
