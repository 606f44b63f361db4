"""Cluster-attention forward pass for NVIDIA B200 (sm_100a).

The computation lives in ``libclusterattn.so`` (hand-written CUDA kernels
behind the C ABI declared in ``include/clusterattn.h``); this package holds
the ctypes binding, the in-tree build script and the seeded input generator.
"""

from ._lib import ClusterAttnError, forward, forward_ex, forward_host, load, sync_status  # noqa: F401

__all__ = ["forward", "forward_ex", "forward_host", "load", "sync_status", "ClusterAttnError"]
