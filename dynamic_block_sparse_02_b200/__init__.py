"""Dynamic top-k block-sparse causal attention (prefill) for NVIDIA B200.

The computation runs in libdsa.so (CUDA kernels for sm_100a behind the C ABI
in include/dsa.h). ``binding`` is its ctypes binding, ``attention`` a small
user-level wrapper, ``workloads`` the named synthetic problem shapes.
The binding is imported lazily, so shape descriptions stay importable on a
machine where the library has not been built yet.
"""
from .workloads import WORKLOADS, WORKLOAD_ORDER, Workload  # noqa: F401

__all__ = ["WORKLOADS", "WORKLOAD_ORDER", "Workload", "BlockSparseAttention"]


def __getattr__(name):
    if name == "BlockSparseAttention":
        from .attention import BlockSparseAttention
        return BlockSparseAttention
    raise AttributeError(name)
