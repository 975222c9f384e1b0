"""MHA2MLA latent-cache decode for B200 (sm_100a).

The compute path is the C-ABI CUDA library built by ``mha_mla_latent_b200.build``
(``lib/libmla_b200.so``); ``mha_mla_latent_b200._lib`` is its ctypes binding and the
names it exports mirror include/mla_api.h.  Attribute access on this package is
forwarded to the binding, which loads the library on first use and raises if it is
missing (there is no CPU fallback).
"""

import importlib

__all__ = ["build", "cache", "convert"]


def __getattr__(name):
    if name.startswith("__") or name in ("build", "cache", "convert", "_lib"):
        return importlib.import_module(f"{__name__}.{name}")
    return getattr(importlib.import_module(f"{__name__}._lib"), name)
