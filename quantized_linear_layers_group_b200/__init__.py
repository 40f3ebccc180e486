"""Quantized linear layers for B200 (sm_100a): dynamic activation quantisation
and a persistent tcgen05 scaled GEMM behind a C ABI (include/qlin.h).

``qlin`` holds the ctypes binding (same names as the C entry points);
``linear`` composes them into the layer a user calls.  Both load libqlin.so
on first use and raise ImportError if it has not been built.
"""
import importlib

__all__ = ["qlin", "linear", "QuantizedLinear", "Workspace", "quantize_weight"]


def __getattr__(name):
    if name in ("qlin", "linear"):
        return importlib.import_module(f".{name}", __name__)
    if name in ("QuantizedLinear", "Workspace", "quantize_weight"):
        return getattr(importlib.import_module(".linear", __name__), name)
    raise AttributeError(name)
