"""B200-native quantized mixture-of-experts layer (Q4_K / Q5_K / Q8_0 experts, Q8_1 activations).

The compute path is the CUDA library ``libmoe.so`` built from ``csrc/`` (C ABI declared in
``include/moe.h``); ``moe`` is its thin ctypes binding.  ``synth`` draws the seeded synthetic
inputs.  Submodules are imported on demand so that loading the input generators does not load
the CUDA library.
"""
import importlib

__all__ = ["moe", "synth", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
