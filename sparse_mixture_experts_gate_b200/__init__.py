"""B200-native (sm_100a) sparse top-k Mixture-of-Experts layer forward.

The layer runs behind the C ABI of include/moe.h (libmoe.so, hand-written CUDA:
router, dispatch, tcgen05 grouped expert GEMM, combine, statistics). This
package holds the CUDA sources (csrc/), the nvcc build (build.py), the ctypes
binding (binding.py) and the seeded synthetic workloads (workloads.py).
"""
from .workloads import WORKLOADS, Workload, make_inputs  # noqa: F401

__all__ = ["WORKLOADS", "Workload", "make_inputs"]
