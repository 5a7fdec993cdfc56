"""Paged single-token decode attention for NVIDIA B200 (sm_100a).

* ``paged_kv_cache_395_b200.pa``: the binding of the C-ABI library ``libpa.so``
  (``include/pa.h``); importing it loads the library and fails loudly if it
  has not been built (``python -m paged_kv_cache_395_b200.build``).
* ``block_manager``: host-side block pool with reference counts and
  copy-on-write.
* ``workloads``: seeded synthetic inputs of the paged decode study.
"""
__all__ = ["block_manager", "workloads", "pa", "build"]
