"""B200-native single-GPU MoE layer (router -> top-k + aux -> permute ->
grouped SwiGLU expert GEMMs -> unpermute), as a C-ABI CUDA library.

The entry points (moe_router_topk, moe_permute, moe_grouped_gemm_fwd/bwd,
moe_unpermute, moe_layer_fwd/bwd, ...) live in libmoe_b200.so, declared in
include/moe.h. This package is a thin ctypes binding with the same names
(argument marshalling only). Attributes are resolved lazily so that the
seeded-input module `synthetic` can be imported without loading the library.
"""
import importlib

__all__ = ["load"]

_SUBMODULES = ("binding", "build", "synthetic")


def __getattr__(name):
    if name.startswith("__") or name in _SUBMODULES:
        if name in _SUBMODULES:
            return importlib.import_module(f"{__name__}.{name}")
        raise AttributeError(name)
    return getattr(importlib.import_module(f"{__name__}.binding"), name)


def load():
    """Load the CUDA library (raises if it is missing or fails to load)."""
    return importlib.import_module(f"{__name__}.binding").load()
