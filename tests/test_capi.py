"""The C-ABI library loads and exports every entry point include/fp8.h
declares; host-side argument checks answer without touching a GPU; the
product path has no route to the oracle and fails loudly without the library."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8.h")
PKG = os.path.join(ROOT, "fp8_mixed_precision_tensor_b200")


@pytest.fixture(scope="module")
def lib():
    from fp8_mixed_precision_tensor_b200 import build

    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(fp8_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("fp8_amax", "fp8_compute_scale", "fp8_cast", "fp8_linear_fwd", "fp8_linear_dgrad",
              "fp8_linear_wgrad", "fp8_adam_step", "fp8_adam_workspace_bytes", "fp8_get_status",
              "fp8_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_symbol_list_matches_header():
    from fp8_mixed_precision_tensor_b200 import fp8

    assert sorted(fp8.SYMBOLS) == declared_functions()


def test_strerror_and_workspace_size(lib):
    lib.fp8_strerror.restype = ctypes.c_char_p
    assert lib.fp8_strerror(0) == b"ok"
    assert b"aligned" in lib.fp8_strerror(2)
    lib.fp8_adam_workspace_bytes.restype = ctypes.c_size_t
    assert lib.fp8_adam_workspace_bytes(3) == 3 * 64
    assert lib.fp8_adam_workspace_bytes(0) == 0


def test_host_side_validation_without_gpu(lib):
    p, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    lib.fp8_amax.argtypes = [p, i, sz, p, p]
    lib.fp8_cast.argtypes = [p, i, sz, i, p, p, p]
    lib.fp8_compute_scale.argtypes = [p, i, i, f, p, p, p]
    lib.fp8_linear_fwd.argtypes = [p, p, p, p, p, i, p, i, p, i, i, i, p]
    fake = 0x10000  # never dereferenced: every call below fails its host checks first
    assert lib.fp8_amax(fake, 1, 10, None, None) == 1                # null amax
    assert lib.fp8_amax(fake, 9, 10, fake, None) == 1                # bad dtype
    assert lib.fp8_amax(fake + 2, 1, 10, fake, None) == 2            # unaligned
    assert lib.fp8_cast(fake, 1, 10, 5, fake, fake, None) == 1       # bad format
    assert lib.fp8_cast(fake, 1, 10, 0, fake, fake + 8, None) == 2   # unaligned output
    assert lib.fp8_compute_scale(fake, 0, 0, 3.0, fake, fake, None) == 1   # mu not a power of two
    assert lib.fp8_compute_scale(fake, 0, -1, 1.0, fake, fake, None) == 1  # negative margin
    # GEMM dims that are not multiples of 16
    assert lib.fp8_linear_fwd(fake, fake, fake, fake, None, 0, fake, 0, None, 32, 32, 24, None) == 3
    assert lib.fp8_linear_fwd(fake, fake, fake, fake, None, 0, fake, 7, None, 32, 32, 32, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    from fp8_mixed_precision_tensor_b200 import fp8

    saved = fp8._lib
    fp8._lib = None
    try:
        with pytest.raises(ImportError):
            fp8.load_library(str(tmp_path / "missing.so"))
    finally:
        fp8._lib = saved


def test_product_never_touches_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"\boracle\b", text), f"{fn} mentions the oracle"


def test_host_side_validation_of_the_next_rows(lib):
    """Scaling variants, FP8 all-reduce, mu rule and sharded Adam entry points
    reject bad arguments on the host, before any device work."""
    p, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    fake = 0x10000
    lib.fp8_amax_scale_cast.argtypes = [p, i, sz, i, p, i, f, p, p, p, p]
    assert lib.fp8_amax_scale_cast(fake, 1, 32, 0, fake, 0, 3.0, fake, fake, fake, None) == 1   # mu
    assert lib.fp8_amax_scale_cast(fake, 1, 32, 0, None, 0, 1.0, fake, fake, fake, None) == 1   # no amax
    assert lib.fp8_amax_scale_cast(fake + 8, 1, 32, 0, fake, 0, 1.0, fake, fake, fake, None) == 2  # unaligned
    lib.fp8_cast_count.argtypes = [p, i, sz, i, p, p, p, p]
    assert lib.fp8_cast_count(fake, 1, 32, 0, fake, fake, None, None) == 1       # no counters
    lib.fp8_grad_cast.argtypes = [p, i, sz, i, p, i, p, p, p, p, p, p]
    assert lib.fp8_grad_cast(fake, 0, 32, 2, fake, 0, fake, fake, fake, fake, None, None) == 1  # FP16 payload
    assert lib.fp8_grad_cast(fake, 0, 32, 1, fake, 0, None, fake, fake, fake, None, None) == 1  # no mu
    lib.fp8_sum_codes.argtypes = [p, i, sz, sz, i, p, p, p, p, p]
    assert lib.fp8_sum_codes(fake, 0, 32, 32, 1, fake, None, None, None, None) == 1      # no ranks
    assert lib.fp8_sum_codes(fake, 2, 40, 32, 1, fake, None, None, None, None) == 2      # ld % 16
    assert lib.fp8_sum_codes(fake, 2, 32, 48, 1, fake, None, None, None, None) == 1      # n > ld
    assert lib.fp8_sum_codes(fake, 5000, 32, 32, 1, fake, None, None, None, None) == 1   # too many ranks

    from fp8_mixed_precision_tensor_b200 import fp8

    lib.fp8_mu_update.argtypes = [p, p, p, ctypes.c_ulonglong, ctypes.POINTER(fp8._MuRule), p]
    bad = fp8._MuRule(1e-3, 10, 3.0, 4.0)   # mu_min not a power of two
    assert lib.fp8_mu_update(fake, fake, fake, 100, ctypes.byref(bad), None) == 1
    bad = fp8._MuRule(1e-3, 0, 0.5, 1.0)    # interval 0
    assert lib.fp8_mu_update(fake, fake, fake, 100, ctypes.byref(bad), None) == 1

    arr = (fp8._Chunk * 1)()
    arr[0] = fp8._Chunk(fake, fake, fake, fake, fake, fake, fake, fake, 64, fake, None, None, None)
    hp = fp8._HParams(1e-4, 0.9, 0.95, 1e-8, 1, 0)
    for name in ("fp8_adam_stats", "fp8_adam_apply"):
        fn = getattr(lib, name)
        fn.argtypes = [ctypes.POINTER(fp8._Chunk), i, ctypes.POINTER(fp8._HParams), p, sz, p]
        assert fn(arr, 1, ctypes.byref(hp), fake, 64, None) == 1   # tracked amax in a sharded half
    arr[0] = fp8._Chunk(fake, fake, fake, fake, fake, fake, fake, fake, 64, None, None, fake, fake)
    lib.fp8_adam_step.argtypes = [ctypes.POINTER(fp8._Chunk), i, ctypes.POINTER(fp8._HParams), p, sz, p]
    assert lib.fp8_adam_step(arr, 1, ctypes.byref(hp), fake, 64, None) == 1  # copy asked for, no codes


def test_adam_rejects_hyper_parameters_outside_the_argued_range(lib):
    """eps below 2^-39 (eps = 0 included) or above 2^64, a non-finite lr or eps,
    beta >= 1 and step 0 are refused on the host with FP8_ERR_INVALID_ARG,
    nothing enqueued."""
    from fp8_mixed_precision_tensor_b200 import fp8

    p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    fake = 0x10000
    arr = (fp8._Chunk * 1)()
    arr[0] = fp8._Chunk(fake, fake, fake, fake, fake, fake, fake, fake, 64, None, None, None, None)
    lib.fp8_adam_step.argtypes = [ctypes.POINTER(fp8._Chunk), i, ctypes.POINTER(fp8._HParams), p, sz, p]
    inf = float("inf")
    for lr, b1, b2, eps, t in ((1e-4, 0.9, 0.95, 0.0, 1), (1e-4, 0.9, 0.95, 2.0 ** -40, 1),
                               (1e-4, 0.9, 0.95, inf, 1), (1e-4, 0.9, 0.95, 2.0 ** 65, 1),
                               (inf, 0.9, 0.95, 1e-8, 1),
                               (1e-4, 1.0, 0.95, 1e-8, 1), (1e-4, 0.9, 0.95, 1e-8, 0)):
        hp = fp8._HParams(lr, b1, b2, eps, t, 0)
        assert lib.fp8_adam_step(arr, 1, ctypes.byref(hp), fake, 64, None) == fp8.FP8_ERR_INVALID_ARG, \
            (lr, b1, b2, eps, t)


def test_adam_step_into_rejects_missing_or_aliased_destinations(lib):
    """The out-of-place step refuses, on the host and before any launch, a
    NULL dest array, a dest with a NULL buffer, a dest buffer that is the
    chunk's own m, v, w or gradient (the inputs must survive the first pass),
    and an unaligned dest."""
    from fp8_mixed_precision_tensor_b200 import fp8

    p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    G, M, V, W, S = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    arr = (fp8._Chunk * 1)()
    arr[0] = fp8._Chunk(G, S, M, S, V, S, W, S, 64, None, None, None, None)
    hp = fp8._HParams(1e-4, 0.9, 0.95, 1e-8, 1, 0)
    fn = lib.fp8_adam_step_into
    fn.argtypes = [ctypes.POINTER(fp8._Chunk), ctypes.POINTER(fp8._Dest), i, ctypes.POINTER(fp8._HParams), p,
                   sz, p]
    assert fn(arr, None, 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG
    dst = (fp8._Dest * 1)()
    for d in ((0x60000, None, 0x80000), (M, 0x70000, 0x80000), (0x60000, V, 0x80000), (0x60000, 0x70000, W),
              (G, 0x70000, 0x80000)):
        dst[0] = fp8._Dest(*d)
        assert fn(arr, dst, 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG, d
    dst[0] = fp8._Dest(0x60008, 0x70000, 0x80000)
    assert fn(arr, dst, 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_UNALIGNED
    # the sharded halves: the same checks, and no tracked master amax
    dst[0] = fp8._Dest(0x60000, 0x70000, 0x80000)
    for name in ("fp8_adam_stats_into", "fp8_adam_apply_into"):
        half = getattr(lib, name)
        half.argtypes = fn.argtypes
        assert half(arr, None, 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG
        arr[0] = fp8._Chunk(G, S, M, S, V, S, W, S, 64, S, None, None, None)
        assert half(arr, dst, 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG
        arr[0] = fp8._Chunk(G, S, M, S, V, S, W, S, 64, None, None, None, None)
        assert half(arr, dst, 1, ctypes.byref(hp), S, 32, None) == fp8.FP8_ERR_INVALID_ARG  # workspace


def test_adam_castgrad_rejects_bad_arguments_on_the_host(lib):
    """The step with the gradient cast in its pass: a NULL gc or amax array, a
    NULL amax entry, a bad mu or margin are refused before any launch."""
    from fp8_mixed_precision_tensor_b200 import fp8

    p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    G, M, V, W, S = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    arr = (fp8._Chunk * 1)()
    arr[0] = fp8._Chunk(G, S, M, S, V, S, W, S, 64, None, None, None, None)
    dst = (fp8._Dest * 1)()
    dst[0] = fp8._Dest(0x60000, 0x70000, 0x80000)
    hp = fp8._HParams(1e-4, 0.9, 0.95, 1e-8, 1, 0)
    fn = lib.fp8_adam_step_into_castgrad
    fn.argtypes = [ctypes.POINTER(fp8._Chunk), ctypes.POINTER(fp8._Dest), ctypes.POINTER(fp8._GradCast), i,
                   ctypes.POINTER(fp8._HParams), p, sz, p]
    amax = (ctypes.c_void_p * 1)(S)
    none = (ctypes.c_void_p * 1)(None)
    good = fp8._GradCast(ctypes.cast(amax, ctypes.POINTER(ctypes.c_void_p)), 1024.0, 0)
    assert fn(arr, dst, None, 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG
    assert fn(arr, None, ctypes.byref(good), 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG
    for gc in (fp8._GradCast(None, 1024.0, 0), fp8._GradCast(ctypes.cast(none, ctypes.POINTER(ctypes.c_void_p)), 1024.0, 0),
               fp8._GradCast(ctypes.cast(amax, ctypes.POINTER(ctypes.c_void_p)), 3.0, 0),
               fp8._GradCast(ctypes.cast(amax, ctypes.POINTER(ctypes.c_void_p)), 1024.0, 65)):
        assert fn(arr, dst, ctypes.byref(gc), 1, ctypes.byref(hp), S, 64, None) == fp8.FP8_ERR_INVALID_ARG


def test_reciprocal_selftest_rejects_bad_arguments_on_the_host(lib):
    fn = lib.fp8_selftest_step_reciprocal
    fn.argtypes = [ctypes.c_uint, ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fake = 0x10000
    assert fn(16, 16, fake, fake, None) == 1           # empty range
    assert fn(0, (1 << 32) + 1, fake, fake, None) == 1  # beyond the 2^32 patterns
    assert fn(0, 16, None, fake, None) == 1            # no counter


def test_encode_selftest_rejects_bad_arguments_on_the_host(lib):
    fn = lib.fp8_selftest_encode
    fn.argtypes = [ctypes.c_int, ctypes.c_uint, ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    fake = 0x10000
    assert fn(2, 0, 16, fake, fake, None) == 1              # FP16 is not an FP8 format
    assert fn(0, 16, 16, fake, fake, None) == 1             # empty range
    assert fn(1, 0, (1 << 32) + 1, fake, fake, None) == 1   # beyond the 2^32 patterns
    assert fn(0, 0, 16, fake, None, None) == 1              # no first-pattern output


def test_wait_selftest_rejects_limits_outside_its_range(lib):
    lib.fp8_selftest_wait_timeout.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    assert lib.fp8_selftest_wait_timeout(0, None) == 1
    assert lib.fp8_selftest_wait_timeout(1000001, None) == 1
