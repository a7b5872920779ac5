"""B200-native PagedAttention decode path.

``libpa.so`` (built from ``csrc/`` for sm_100a) exports the C ABI declared in
``include/pa.h``: ``pa_reshape_and_cache`` (cache write), ``pa_decode``
(paged single-token decode attention, split-K with an in-kernel merge) and
``pa_copy_blocks`` (copy-on-write block copy).  ``binding`` is a thin ctypes
layer over it with the same names; it only marshals arguments.

The native library is loaded on first call and there is no fallback: if it
is missing or no CUDA device is present, the call raises.
"""
from . import accounting, binding, workloads  # noqa: F401

__all__ = ["accounting", "binding", "workloads"]
