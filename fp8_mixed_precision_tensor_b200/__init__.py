"""B200-native FP8 mixed-precision training hot path.

The compute lives in ``libfp8.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/fp8.h``).  ``fp8_mixed_precision_tensor_b200.fp8``
is the thin ctypes binding with the same entry-point names; it is a separate
submodule so that the seeded input generators in ``synth`` load without a GPU
or a built library.
"""
