"""Kimi Delta Attention (KDA) prefill and decode for B200 (sm_100a).

The compute lives in ``libkda.so`` (hand-written CUDA behind a C ABI, see
``include/kda.h``); ``binding`` marshals arguments to it with ctypes.
The binding is imported lazily so that ``inputs`` (seeded synthetic data)
can be used without touching the CUDA library.
"""
from __future__ import annotations

__all__ = ["binding", "inputs", "kda_chunk_prefill", "kda_decode_step",
           "kda_chunk_prefill_workspace_bytes"]


def __getattr__(name):
    if name in ("kda_chunk_prefill", "kda_decode_step",
                "kda_chunk_prefill_workspace_bytes"):
        from . import binding
        return getattr(binding, name)
    if name in ("binding", "inputs"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
