"""Grouped-query causal attention (q/k RMSNorm -> RoPE -> causal GQA SDPA) for B200.

The compute lives in ``libgqa_attn.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/gqa_attn.h``).  ``binding`` marshals torch tensors into that
ABI.  Submodules load on first access, so ``synthetic`` can be used without
loading the CUDA library.
"""
import importlib

__all__ = ["binding", "synthetic"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
