"""Attention states over sequence partitions with cached-state reuse, for B200.

The compute path is the CUDA library ``libasp.so`` (C ABI in
include/as_partition.h) reached through :mod:`.api`; :mod:`.workloads` holds
the seeded input generators.  Importing :mod:`.api` fails if the library has
not been built (``python -m attention_state_reuse_partition_b200.build``).
"""
__version__ = "0.1.0"
