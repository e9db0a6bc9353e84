"""B200-native forward pass of one sparse Mixture-of-Experts layer.

The compute lives in ``libmoe.so`` (hand-written sm_100a CUDA kernels behind a
C ABI declared in ``include/moe.h``); ``_lib`` is a thin ctypes binding with the
same entry-point names. Importing the binding loads the library and raises if it
is missing: there is no CPU fallback.

``inputs`` (seeded synthetic workloads) is importable without the library.
"""

__all__ = ["moe_route", "moe_permute", "moe_expert_ffn", "moe_unpermute", "moe_forward",
           "moe_forward_host", "moe_mxfp8_quantize", "moe_mxfp4_quantize",
           "moe_forward_workspace_size", "MoEError", "inputs"]


def __getattr__(name):
    if name in __all__ and name != "inputs":
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
