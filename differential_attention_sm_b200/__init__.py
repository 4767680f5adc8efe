"""Differential attention (V1 and V2) for NVIDIA B200 (sm_100a).

The operator (softmax(Q1 K1^T / sqrt d) - lambda softmax(Q2 K2^T / sqrt d)) V
runs in hand-written CUDA kernels behind a C ABI (``libdiffattn.so``, see
``include/diffattn.h``).  ``differential_attention_sm_b200.binding`` is a thin
ctypes layer over that library with the same function names; it only
marshals arguments.  ``differential_attention_sm_b200.inputs`` draws seeded
synthetic inputs.  Nothing here falls back to a CPU implementation: if the
library cannot be loaded, the binding raises.
"""
import importlib

__all__ = ["binding", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
