"""B200-native routed Mixture-of-Experts FFN (sm_100a).

The layer runs as hand-written CUDA kernels behind the C ABI declared in
``include/moe.h`` (``libmoe_b200.so``, built in-tree).  ``api`` is the thin
ctypes binding with the same entry-point names; ``workloads`` draws seeded
synthetic inputs.  Importing the package does not load the library: the
binding loads it on first use and raises if it is missing.
"""

__all__ = ["api", "workloads"]
