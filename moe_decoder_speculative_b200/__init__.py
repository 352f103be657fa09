"""B200-native greedy MoE speculative-verify step (jina-ocr-v1 decoder shape).

The compute lives in a C-ABI shared library of hand-written sm_100a CUDA
kernels (``csrc/``, declared in ``include/moe_verify.h``).  ``binding`` is the
thin ctypes layer over it; ``workloads`` draws the seeded synthetic inputs.
Importing this package does not load the CUDA library; the first call into
``binding`` does, and fails loudly if it is missing.
"""
import importlib

__all__ = ["binding", "workloads", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
