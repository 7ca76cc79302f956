"""TurboQuant KV-cache codec and fused decode attention for NVIDIA B200 (sm_100a).

``turboquant_kv_cache_rht_b200.tq`` is the Python binding of the C-ABI library
``libtq.so`` (built in-tree by ``turboquant_kv_cache_rht_b200.build``); importing
it loads the library and fails loudly if it is missing.
``turboquant_kv_cache_rht_b200.workloads`` holds the seeded synthetic inputs.
"""
__all__ = ["tq", "workloads"]
