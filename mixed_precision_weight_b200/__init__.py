"""DV-SSQ compressed linear layer for B200 (sm_100a).

The CUDA library and its ctypes binding live in ``binding``; attribute access
on this package (``mixed_precision_weight_b200.dvssq_encode`` and so on)
imports it on first use and fails loudly if libdvssq.so is missing.  The
seeded input generators (``synth``) need no GPU library.
"""
import importlib

__all__ = ["binding", "synth", "build"]


def __getattr__(name):
    if name in ("binding", "synth", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    binding = importlib.import_module(f"{__name__}.binding")
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
