"""libw4a4: DSFQ W4A4 quantized linear layer for NVIDIA B200 (sm_100a).

The compute lives in the CUDA shared library libw4a4.so (C ABI declared in
include/w4a4.h).  ``w4a4_post_quantized_b200.w4a4`` is the thin ctypes binding
with the same names; it raises ImportError when the library is missing, and
there is no fallback path.  ``synth`` generates seeded VGGT-shaped inputs.
"""
import importlib

__all__ = ["w4a4", "synth"]


def __getattr__(name):
    if name in ("w4a4", "synth"):
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
