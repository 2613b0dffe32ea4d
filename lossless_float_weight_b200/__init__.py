"""B200-native ZipNN-style lossless codec for BF16, FP32 and FP8 (E4M3) tensors.

The codec itself lives in the CUDA library ``libzipnn_b200.so`` behind the C ABI of
``include/zipnn.h``; :mod:`lossless_float_weight_b200.zipnn` is the thin Python binding
over it. The binding is imported on first use of one of its names, so that the seeded
input generators in :mod:`lossless_float_weight_b200.workloads` stay importable on a
machine where the library has not been built.
"""
import importlib

_SUBMODULES = ("workloads", "zipnn", "build")


def __getattr__(name):
    if name.startswith("_") or name in _SUBMODULES:
        raise AttributeError(name)
    return getattr(importlib.import_module(__name__ + ".zipnn"), name)
