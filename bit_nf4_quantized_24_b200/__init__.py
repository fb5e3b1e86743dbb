"""QLoRA frozen-NF4 linear layer for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libqlora_nf4.so`` (hand-written CUDA
kernels, declared in ``include/qlora_nf4.h``).  ``binding`` is a thin ctypes
layer over it that marshals torch CUDA tensors; it raises if the library is
missing -- there is no CPU fallback.  ``workloads`` draws the seeded inputs.
"""
import importlib

__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
