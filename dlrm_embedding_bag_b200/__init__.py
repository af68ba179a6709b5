"""DLRMv1 sparse/interaction stage on B200 (sm_100a).

The compute path is a C-ABI shared library of hand-written CUDA kernels
(``libdlrm_sparse.so``, declared in ``include/dlrm_sparse.h``); ``ops`` is the
thin Python binding over it. The library is loaded on first use and its
absence is an error: there is no CPU fallback.
"""
from . import synthetic  # noqa: F401  (input generator, no CUDA needed)

__all__ = ["synthetic", "ops"]


def __getattr__(name):
    if name == "ops":
        from . import ops

        return ops
    raise AttributeError(name)
