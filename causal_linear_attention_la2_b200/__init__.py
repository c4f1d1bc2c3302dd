"""Lightning Attention-2 (causal linear attention with per-head decay) for B200.

The compute path is the CUDA library ``libla2.so`` (sm_100a kernels behind a C
ABI declared in ``include/la2.h``); ``la2`` is its thin ctypes binding.  The
binding is loaded lazily so that ``inputs`` can be imported on machines
without a GPU.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs"]
