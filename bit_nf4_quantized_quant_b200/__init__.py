"""QLoRA frozen-NF4 linear layer for B200 (sm_100a).

The compute path lives in ``libqlora_nf4.so`` (hand-written CUDA behind a
C ABI declared in ``include/qlora_nf4.h``); ``ops`` is a thin ctypes binding
with the same names.  Importing the package does not load the library;
calling any op does, and fails loudly if it is missing.
"""

__all__ = ["ops", "inputs"]


def __getattr__(name):
    if name == "ops":
        from . import _ops as ops
        return ops
    raise AttributeError(name)
