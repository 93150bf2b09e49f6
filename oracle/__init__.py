"""CPU oracle for the FP8 mixed-precision training hot path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use it; the product path never does.  It wraps the plain C
file ``fp8_oracle.c`` (float64 arithmetic, OpenMP loops) and shares no code
with the CUDA library.  Sources are cited in the C file:

* "FP8-LM: Training FP8 Large Language Models" (paper memo), 提案手法 O1
  (Eq. 3, gradient auto-scaling) and O2 (precision-decoupled Adam).
* "Training and inference of large language models using 8-bit floating
  point" (paper review), 제안 방법 (per-tensor amax scaling, E4M3/E5M2, scale
  before the cast and undo after the matmul).

Every function is pinned by ``tests/test_oracle_pins.py`` against the format
definitions, closed forms, brute force and independent library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

E4M3, E5M2, F16 = 0, 1, 2
DT_F32, DT_BF16, DT_F16 = 0, 1, 2
OK, ERR_NONFINITE = 0, 6

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile fp8_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _bind(lib):
    d, i, u, sz, p = ctypes.c_double, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_void_p
    ll = ctypes.c_longlong
    lib.orc_fp8_decode.argtypes, lib.orc_fp8_decode.restype = [i, u], d
    lib.orc_f16_decode.argtypes, lib.orc_f16_decode.restype = [u], d
    lib.orc_fp8_encode.argtypes, lib.orc_fp8_encode.restype = [i, d], u
    lib.orc_f16_encode.argtypes, lib.orc_f16_encode.restype = [d], u
    lib.orc_fmt_max.argtypes, lib.orc_fmt_max.restype = [i], d
    lib.orc_amax.argtypes, lib.orc_amax.restype = [p, i, sz], d
    lib.orc_amax_parallel.argtypes, lib.orc_amax_parallel.restype = [p, i, sz], d
    lib.orc_floor_log2_ratio.argtypes, lib.orc_floor_log2_ratio.restype = [d, d], i
    lib.orc_compute_scale.argtypes, lib.orc_compute_scale.restype = [d, i, i, ctypes.POINTER(d)], i
    lib.orc_compute_scale_mu.argtypes = [d, i, i, d, ctypes.POINTER(d)]
    lib.orc_compute_scale_mu.restype = i
    lib.orc_cast.argtypes, lib.orc_cast.restype = [p, i, sz, i, d, p], None
    lib.orc_gemm.argtypes = [p, i, ll, ll, d, p, i, ll, ll, d, p, i, i, i, p, p]
    lib.orc_gemm.restype = None
    lib.orc_gemm_sampled.argtypes = [p, i, ll, ll, d, p, i, ll, ll, d, p, i, p, p, ll, p, p]
    lib.orc_gemm_sampled.restype = None
    lib.orc_adam_update_f64.argtypes = [sz, p, p, p, p, d, d, d, d, i, p, p, p]
    lib.orc_adam_update_f64.restype = None
    lib.orc_adam_step.argtypes = [sz, p, d, p, ctypes.POINTER(d), p, ctypes.POINTER(d), p,
                                  ctypes.POINTER(d), d, d, d, d, i, i, p, p]
    lib.orc_adam_step.restype = i
    lib.orc_adam_step_amax.argtypes = [sz, p, d, p, ctypes.POINTER(d), p, ctypes.POINTER(d), p,
                                       ctypes.POINTER(d), d, d, d, d, i, i, p, p, p]
    lib.orc_adam_step_amax.restype = i
    u64p = ctypes.POINTER(ctypes.c_ulonglong)
    lib.orc_cast_counts.argtypes, lib.orc_cast_counts.restype = [p, i, sz, i, d, p, u64p], None
    lib.orc_grad_scale.argtypes, lib.orc_grad_scale.restype = [d, i, i, d, ctypes.POINTER(d)], i
    lib.orc_sum_codes.argtypes, lib.orc_sum_codes.restype = [p, i, sz, sz, i, p, u64p], None
    lib.orc_mu_update.argtypes = [ctypes.POINTER(d), ctypes.POINTER(i), ctypes.c_ulonglong, ctypes.c_ulonglong,
                                  d, i, d, d]
    lib.orc_mu_update.restype = None
    lib.orc_num_threads.argtypes, lib.orc_num_threads.restype = [], i
    lib.orc_set_num_threads.argtypes, lib.orc_set_num_threads.restype = [i], None
    return lib


class use_library:
    """Context manager: route this module's calls to another build of the
    oracle (the mutation tests load deliberately broken copies)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _dtype_code(x: np.ndarray, dtype: int | None) -> int:
    if dtype is not None:
        return dtype
    if x.dtype == np.float32:
        return DT_F32
    raise ValueError("uint16 inputs need an explicit dtype (DT_BF16 or DT_F16)")


# ---------------------------------------------------------------- formats
def decode(fmt: int, code: int) -> float:
    """Value of one E4M3/E5M2 code, from the bit-field definition."""
    return _load().orc_fp8_decode(fmt, code)


def decode_table(fmt: int) -> np.ndarray:
    """All 256 code values of an FP8 format."""
    return np.array([decode(fmt, c) for c in range(256)], dtype=np.float64)


def f16_decode(bits: int) -> float:
    return _load().orc_f16_decode(bits)


def encode(fmt: int, y: float) -> int:
    """RNE, saturating encode of one real number (E4M3/E5M2)."""
    return _load().orc_fp8_encode(fmt, float(y))


def f16_encode(y: float) -> int:
    return _load().orc_f16_encode(float(y))


def fmt_max(fmt: int) -> float:
    return _load().orc_fmt_max(fmt)


# ---------------------------------------------------------------- amax / scale / cast
def amax(x: np.ndarray, dtype: int | None = None, parallel: bool = False) -> float:
    """max_i |x_i| of a contiguous fp32 / bf16-bits / fp16-bits array."""
    x = np.ascontiguousarray(x)
    f = _load().orc_amax_parallel if parallel else _load().orc_amax
    return f(_ptr(x), _dtype_code(x, dtype), x.size)


def floor_log2_ratio(amax_value: float, fmt_max_value: float) -> int:
    return _load().orc_floor_log2_ratio(float(amax_value), float(fmt_max_value))


def compute_scale(amax_value: float, fmt: int, margin: int, mu: float = 1.0) -> tuple[int, float]:
    """(status, total scale) with total scale = mu * 2^(floor(log2(fmt_max/(mu*amax))) - margin)."""
    out = ctypes.c_double()
    rc = _load().orc_compute_scale_mu(float(amax_value), fmt, margin, float(mu), ctypes.byref(out))
    return rc, out.value


def cast(x: np.ndarray, fmt: int, scale: float, dtype: int | None = None) -> np.ndarray:
    """q_i = enc(x_i * scale); uint8 codes, or uint16 half bits for F16."""
    x = np.ascontiguousarray(x)
    q = np.empty(x.shape, dtype=np.uint16 if fmt == F16 else np.uint8)
    _load().orc_cast(_ptr(x), _dtype_code(x, dtype), x.size, fmt, float(scale), _ptr(q))
    return q


# ---------------------------------------------------------------- GEMMs
def _gemm(A, fa, a_si, a_sk, inv_sa, B, fb, b_sj, b_sk, inv_sb, bias, M, N, K, samples=None):
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    bias_p = None
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float64)
        bias_p = _ptr(bias)
    lib = _load()
    if samples is None:
        C = np.empty((M, N), dtype=np.float64)
        Cabs = np.empty((M, N), dtype=np.float64)
        lib.orc_gemm(_ptr(A), fa, a_si, a_sk, inv_sa, _ptr(B), fb, b_sj, b_sk, inv_sb, bias_p,
                     M, N, K, _ptr(C), _ptr(Cabs))
        return C, Cabs
    rows = np.ascontiguousarray(samples[0], dtype=np.int32)
    cols = np.ascontiguousarray(samples[1], dtype=np.int32)
    C = np.empty(rows.size, dtype=np.float64)
    Cabs = np.empty(rows.size, dtype=np.float64)
    lib.orc_gemm_sampled(_ptr(A), fa, a_si, a_sk, inv_sa, _ptr(B), fb, b_sj, b_sk, inv_sb, bias_p,
                         K, _ptr(rows), _ptr(cols), rows.size, _ptr(C), _ptr(Cabs))
    return C, Cabs


def linear_fwd(xq, x_inv, wq, w_inv, M, N, K, bias=None, samples=None, fmt_x=E4M3, fmt_w=E4M3):
    """Y[M,N] = (Xq[M,K] . Wq[N,K]^T) * x_inv * w_inv (+ bias).  Returns (Y, sum|a b|)."""
    return _gemm(xq, fmt_x, K, 1, x_inv, wq, fmt_w, K, 1, w_inv, bias, M, N, K, samples)


def linear_dgrad(dyq, dy_inv, wq, w_inv, M, N, K, samples=None, fmt_dy=E5M2, fmt_w=E4M3):
    """dX[M,K] = (dYq[M,N] . Wq[N,K]) * dy_inv * w_inv.  Returns (dX, sum|a b|)."""
    return _gemm(dyq, fmt_dy, N, 1, dy_inv, wq, fmt_w, 1, K, w_inv, None, M, K, N, samples)


def linear_wgrad(dyq, dy_inv, xq, x_inv, M, N, K, samples=None, fmt_dy=E5M2, fmt_x=E4M3):
    """dW[N,K] = (dYq[M,N]^T . Xq[M,K]) * dy_inv * x_inv.  Returns (dW, sum|a b|)."""
    return _gemm(dyq, fmt_dy, 1, N, dy_inv, xq, fmt_x, 1, K, x_inv, None, N, K, M, samples)


# ---------------------------------------------------------------- Adam
def adam_update_f64(g, m0, v0, w0, lr, beta1, beta2, eps, t):
    """The float64 Adam update on decoded values: returns (m, v, w)."""
    arrs = [np.ascontiguousarray(a, dtype=np.float64) for a in (g, m0, v0, w0)]
    n = arrs[0].size
    m, v, w = (np.empty(n) for _ in range(3))
    _load().orc_adam_update_f64(n, *(_ptr(a) for a in arrs), lr, beta1, beta2, eps, t,
                                _ptr(m), _ptr(v), _ptr(w))
    return m, v, w


def adam_step(gq, g_inv, mq, s_m, vh, s_v, wh, s_w, lr, beta1, beta2, eps, t, margin, amax_in=None):
    """One decoupled Adam step on one tensor's stored state (copies; inputs untouched).

    Returns dict(rc, mq, s_m, vh, s_v, wh, s_w, amax=(|m|, v, |w|) of the new float64 values).
    amax_in: optional (|m|, v, |w|) amaxes the new scales are taken from instead
    of this call's own (a slice of a larger tensor, see adam_step_sharded).
    """
    n = np.asarray(gq).size
    gq = np.ascontiguousarray(gq, dtype=np.uint8)
    mq = np.array(mq, dtype=np.uint8, copy=True).reshape(-1)
    vh = np.array(vh, dtype=np.uint16, copy=True).reshape(-1)
    wh = np.array(wh, dtype=np.uint16, copy=True).reshape(-1)
    sm, sv, sw = ctypes.c_double(s_m), ctypes.c_double(s_v), ctypes.c_double(s_w)
    work = np.empty(7 * max(n, 1), dtype=np.float64)
    am = np.zeros(3, dtype=np.float64)
    if amax_in is None:
        rc = _load().orc_adam_step(n, _ptr(gq), float(g_inv), _ptr(mq), ctypes.byref(sm), _ptr(vh),
                                   ctypes.byref(sv), _ptr(wh), ctypes.byref(sw), lr, beta1, beta2, eps,
                                   t, margin, _ptr(work), _ptr(am))
    else:
        ain = np.array(amax_in, dtype=np.float64)
        rc = _load().orc_adam_step_amax(n, _ptr(gq), float(g_inv), _ptr(mq), ctypes.byref(sm), _ptr(vh),
                                        ctypes.byref(sv), _ptr(wh), ctypes.byref(sw), lr, beta1, beta2,
                                        eps, t, margin, _ptr(work), _ptr(ain), _ptr(am))
    return dict(rc=rc, mq=mq, s_m=sm.value, vh=vh, s_v=sv.value, wh=wh, s_w=sw.value,
                amax=tuple(am))


def _nan_max(values):
    r = 0.0
    for x in values:
        if np.isnan(x):
            return float("nan")
        r = max(r, x)
    return r


def adam_step_sharded(gq, g_inv, mq, s_m, vh, s_v, wh, s_w, lr, beta1, beta2, eps, t, margin, bounds):
    """The step of adam_step with the tensor's elements split into slices
    [lo, hi) ("FP8-LM", 提案手法 O3: optimizer state partitioned ZeRO-style
    over data-parallel ranks): every slice first yields the amaxes of its new
    values; the tensor's amax is their maximum (a NaN wins); every slice is
    then requantised with the scales of that maximum.  Returns the
    concatenated state in the form adam_step returns it."""
    gq, mq, vh, wh = (np.asarray(a).reshape(-1) for a in (gq, mq, vh, wh))
    args = (lr, beta1, beta2, eps, t, margin)
    parts = [(lo, hi) for lo, hi in bounds]
    stats = [adam_step(gq[lo:hi], g_inv, mq[lo:hi], s_m, vh[lo:hi], s_v, wh[lo:hi], s_w, *args)["amax"]
             for lo, hi in parts]
    glob = tuple(_nan_max([s[j] for s in stats]) for j in range(3))
    outs = [adam_step(gq[lo:hi], g_inv, mq[lo:hi], s_m, vh[lo:hi], s_v, wh[lo:hi], s_w, *args, amax_in=glob)
            for lo, hi in parts]
    cat = {k: np.concatenate([o[k] for o in outs]) for k in ("mq", "vh", "wh")}
    return dict(rc=max(o["rc"] for o in outs), s_m=outs[0]["s_m"], s_v=outs[0]["s_v"], s_w=outs[0]["s_w"],
                amax=glob, **cat)


def adam_master_e4m3(wh, s_w: float, margin: int):
    """E4M3 copy of a stored FP16 master for the next forward pass ("FP8-LM",
    提案手法 O2 master weights, cast as in "Training and inference of large
    language models using 8-bit floating point", 제안 방법): the dequantised
    master is dec_f16(wh) / s_w; its E4M3 scale s_q comes from its amax with
    fmt_max 448; codes = enc_E4M3(dec_f16(wh) / s_w * s_q), where the product
    s_q / s_w is an exact power of two.  Returns (codes, s_q)."""
    wh = np.ascontiguousarray(wh).view(np.uint16)
    a = amax(wh, DT_F16) / s_w
    rc, s_q = compute_scale(a, E4M3, margin)
    return cast(wh, E4M3, s_q / s_w, DT_F16), s_q


# ---------------------------------------------------------------- scaling variants, FP8 all-reduce
def cast_counts(x, fmt: int, scale: float, dtype: int | None = None):
    """(codes, (underflows, overflows)) of cast(x, fmt, scale)."""
    x = np.ascontiguousarray(x)
    q = np.empty(x.shape, dtype=np.uint16 if fmt == F16 else np.uint8)
    counts = (ctypes.c_ulonglong * 2)(0, 0)
    _load().orc_cast_counts(_ptr(x), _dtype_code(x, dtype), x.size, fmt, float(scale), _ptr(q), counts)
    return q, (counts[0], counts[1])


def grad_scale(amax_value: float, fmt: int, margin: int, mu: float) -> tuple[int, float]:
    """(status, S) with S = mu * 2^(floor(log2(fmt_max/amax)) - margin): the
    shared payload scale of the FP8 gradient all-reduce."""
    out = ctypes.c_double(0.0)
    rc = _load().orc_grad_scale(float(amax_value), fmt, margin, float(mu), ctypes.byref(out))
    return rc, out.value


def sum_codes(rows, fmt: int):
    """rows: [nranks, n] uint8 codes with one shared scale.  Returns (codes of
    the exact sum re-encoded, (underflows, overflows))."""
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    nranks, n = rows.shape
    out = np.empty(n, dtype=np.uint8)
    counts = (ctypes.c_ulonglong * 2)(0, 0)
    _load().orc_sum_codes(_ptr(rows), nranks, n, n, fmt, _ptr(out), counts)
    return out, (counts[0], counts[1])


def mu_update(mu: float, clean: int, overflows: int, n: int, theta: float, interval: int,
              mu_min: float, mu_max: float) -> tuple[float, int]:
    """The auto-scaling rule for mu: returns (mu, clean steps) after one step."""
    m, c = ctypes.c_double(mu), ctypes.c_int(clean)
    _load().orc_mu_update(ctypes.byref(m), ctypes.byref(c), overflows, n, float(theta), interval,
                          float(mu_min), float(mu_max))
    return m.value, c.value


def fp8_allreduce(grads, fmt: int, margin: int, mu: float):
    """The FP8 gradient all-reduce over len(grads) ranks ("FP8-LM", 提案手法
    O1): the amax over all ranks, the shared scale S = grad_scale(amax, mu),
    every rank's payload cast with S, the exact sum of the payloads
    re-encoded at S.  Returns dict(codes, S, rc, cast_counts, sum_counts);
    the reduced gradient is dec(codes) / S (a sum over ranks, not a mean)."""
    grads = [np.ascontiguousarray(g, dtype=np.float32).reshape(-1) for g in grads]
    a = amax(np.stack(grads).reshape(-1)) if grads[0].size else 0.0
    rc, S = grad_scale(a, fmt, margin, mu)
    rows, cc = [], [0, 0]
    for g in grads:
        q, c = cast_counts(g, fmt, S)
        rows.append(q)
        cc[0] += c[0]
        cc[1] += c[1]
    codes, sc = sum_codes(np.stack(rows), fmt)
    return dict(codes=codes, S=S, rc=rc, cast_counts=tuple(cc), sum_counts=sc, payloads=np.stack(rows))


def num_threads() -> int:
    return _load().orc_num_threads()


def set_num_threads(nt: int) -> None:
    _load().orc_set_num_threads(nt)
