"""B200-native Hybrid Sparse Attention (HSA) decode step over paged KV.

The compute path lives in ``libwa.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/wa.h``).  ``linear_attention_paged_b200.wa`` is the thin ctypes
binding with the same function names; importing it loads the library and raises if
it is missing.  ``linear_attention_paged_b200.workloads`` draws seeded inputs.
"""
