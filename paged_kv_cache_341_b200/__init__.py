"""Paged KV cache decode path for NVIDIA B200 (sm_100a).

``paged_kv_cache_341_b200.pa`` is the Python binding of the C-ABI library
``libpagedattn.so`` (header ``include/pa.h``); importing it loads the library
and raises if it has not been built -- there is no CPU fallback.

``paged_kv_cache_341_b200.workloads`` holds only seeded input generators
(lengths, pool orders, random K/V/q values); it performs none of the method's
arithmetic and is importable without the library.

Building: ``python -m paged_kv_cache_341_b200.build`` (or
``__graft_entry__.build()``).
"""
