"""B200-native attention-guided KV-cache eviction and compaction.

The hot path lives in the C-ABI library ``libkvc.so`` (CUDA, sm_100a), built in
this package directory; ``agent_kv_cache_lse_b200.kvc`` is its thin ctypes
binding and ``agent_kv_cache_lse_b200.synth`` draws seeded synthetic workloads.
Importing the package loads nothing; the binding loads the library on first use
and raises if it is missing.
"""
__all__ = ["kvc", "synth"]
