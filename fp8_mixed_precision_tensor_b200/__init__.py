"""B200-native FP8 mixed-precision training hot path.

The compute lives in ``libfp8.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/fp8.h``).  ``fp8_mixed_precision_tensor_b200.fp8``
is the thin ctypes binding with the same entry-point names; it is imported
lazily so that the seeded input generators in ``synth`` load without a GPU.
"""

__all__ = ["fp8", "synth"]


def __getattr__(name):
    if name == "fp8":
        from . import fp8 as _fp8

        return _fp8
    raise AttributeError(name)
