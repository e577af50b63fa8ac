"""SparSTAR per-scale block-sparse attention forward on B200 (sm_100a).

The compute lives in ``libsparstar.so`` (C ABI, declared in
``include/sparstar.h``); ``block_sparse_attention_18_b200.sparstar`` is the thin
Python binding with the same entry-point names.  Importing this package does
not load the library; importing ``.sparstar`` does, and fails loudly when the
library is missing.
"""
__all__ = ["sparstar", "synth"]
