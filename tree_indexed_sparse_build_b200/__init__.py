"""Tree-indexed sparse decode attention on B200 (sm_100a).

A b-ary tree of mean-pooled key summaries over fixed-size leaf blocks of a KV
cache, a top-down beam descent per query, and exact softmax attention over the
tokens of the selected leaves.  The work runs in the CUDA library ``libzha``
(C ABI, ``include/zha.h``); ``zha`` is its thin ctypes binding.
"""
