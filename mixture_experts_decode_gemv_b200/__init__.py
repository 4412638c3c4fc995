"""Decode-time Mixture-of-Experts layer for NVIDIA B200 (sm_100a).

The layer runs in ``libmoedecode.so`` (C ABI in ``include/moe_decode.h``); ``binding`` exposes
its entry points under the same names. Attribute access on this package (``moe_decode_forward``,
``moe_workspace_bytes`` ...) loads the binding on first use, so importing ``synthetic`` alone never
needs the compiled library.
"""
import importlib

__version__ = "0.1.0"
_SUBMODULES = ("binding", "build", "device_layer", "synthetic")


def __getattr__(name):
    if name in _SUBMODULES:
        return importlib.import_module(f"{__name__}.{name}")
    binding = importlib.import_module(f"{__name__}.binding")
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
