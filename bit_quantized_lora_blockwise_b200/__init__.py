"""QLoRA frozen-base linear layer for B200 (sm_100a).

The compute lives in ``libqlora.so`` (hand-written CUDA, C ABI declared in
``include/qlora.h``); ``binding`` marshals torch tensors into that ABI.
Importing the package does not load the library; ``binding`` does, and it
raises if the library is missing (there is no CPU fallback).
"""
__all__ = ["binding", "inputs"]


def __getattr__(name):
    if name in ("binding", "inputs"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
