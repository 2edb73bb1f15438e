"""B200-native asymmetric KV merging (KVSlimmer) hot path.

Submodules:
  kvs         -- ctypes binding of the C-ABI library libkvs.so (CUDA kernels)
  inputs      -- seeded synthetic workloads (no merging arithmetic)
  accounting  -- cache and roofline byte counts

Importing the package loads nothing; ``from asymmetric_kv_merging_b200 import kvs``
loads the CUDA library and fails loudly if it is missing.
"""
