"""ctypes binding of libfp8 (the C ABI in include/fp8.h).

Argument marshalling only: every function takes torch tensors that already
live on the current CUDA device, passes their data pointers, sizes and the
current stream to the entry point of the same name, and raises FP8Error on a
non-zero status.  All arithmetic happens in the CUDA kernels of libfp8.so;
there is no fallback, and importing this module fails loudly when the library
has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8.so")

# status codes / enums (include/fp8.h)
FP8_OK, FP8_ERR_INVALID_ARG, FP8_ERR_UNALIGNED, FP8_ERR_UNSUPPORTED = 0, 1, 2, 3
FP8_ERR_CUDA, FP8_ERR_TIMEOUT, FP8_ERR_NONFINITE = 4, 5, 6
FP8_STATUS_NONFINITE, FP8_STATUS_TIMEOUT, FP8_STATUS_INTERNAL, FP8_STATUS_BAD_MU = 1, 2, 4, 8
FP8_DT_F32, FP8_DT_BF16, FP8_DT_F16 = 0, 1, 2
FP8_DT_BF16_RTO = 3  # GEMM outputs only: bfloat16 rounded to odd, for a following FP8 cast
FP8_E4M3, FP8_E5M2, FP8_F16S = 0, 1, 2

_DT = {torch.float32: FP8_DT_F32, torch.bfloat16: FP8_DT_BF16, torch.float16: FP8_DT_F16}

SYMBOLS = ("fp8_amax", "fp8_compute_scale", "fp8_cast", "fp8_scale_cast", "fp8_amax_scale_cast", "fp8_cast_count",
           "fp8_grad_cast",
           "fp8_sum_codes", "fp8_mu_update", "fp8_linear_fwd", "fp8_linear_dgrad",
           "fp8_linear_wgrad", "fp8_adam_workspace_bytes", "fp8_adam_step", "fp8_adam_stats",
           "fp8_adam_apply", "fp8_adam_step_noalloc", "fp8_adam_step_into", "fp8_adam_step_into_castgrad",
           "fp8_adam_stats_into",
           "fp8_adam_apply_into",
           "fp8_selftest_wait_timeout", "fp8_selftest_step_reciprocal", "fp8_selftest_encode", "fp8_get_status", "fp8_strerror")


class FP8Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {fp8_strerror(code)} (status {code})")
        self.code = code


class _Chunk(ctypes.Structure):
    _fields_ = [("g", ctypes.c_void_p), ("g_inv", ctypes.c_void_p), ("m", ctypes.c_void_p),
                ("m_scale", ctypes.c_void_p), ("v", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("w_scale", ctypes.c_void_p), ("n", ctypes.c_size_t),
                ("w_amax", ctypes.c_void_p), ("wq", ctypes.c_void_p), ("wq_scale", ctypes.c_void_p),
                ("wq_inv", ctypes.c_void_p)]


class _Dest(ctypes.Structure):
    _fields_ = [("m", ctypes.c_void_p), ("v", ctypes.c_void_p), ("w", ctypes.c_void_p)]


class _GradCast(ctypes.Structure):
    _fields_ = [("amax", ctypes.POINTER(ctypes.c_void_p)), ("mu", ctypes.c_float), ("margin", ctypes.c_int)]


class _MuRule(ctypes.Structure):
    _fields_ = [("theta", ctypes.c_float), ("interval", ctypes.c_int), ("mu_min", ctypes.c_float),
                ("mu_max", ctypes.c_float)]


class _HParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("step", ctypes.c_int), ("margin", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfp8.so and declare the signatures of every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libfp8.so not built ({path}); run python -m fp8_mixed_precision_tensor_b200.build")
    lib = ctypes.CDLL(path)
    p, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    lib.fp8_amax.argtypes = [p, i, sz, p, p]
    lib.fp8_compute_scale.argtypes = [p, i, i, f, p, p, p]
    lib.fp8_cast.argtypes = [p, i, sz, i, p, p, p]
    lib.fp8_scale_cast.argtypes = [p, i, sz, i, p, i, f, p, p, p, p]
    lib.fp8_amax_scale_cast.argtypes = [p, i, sz, i, p, i, f, p, p, p, p]
    lib.fp8_cast_count.argtypes = [p, i, sz, i, p, p, p, p]
    lib.fp8_grad_cast.argtypes = [p, i, sz, i, p, i, p, p, p, p, p, p]
    lib.fp8_sum_codes.argtypes = [p, i, sz, sz, i, p, p, p, p, p]
    lib.fp8_mu_update.argtypes = [p, p, p, ctypes.c_ulonglong, ctypes.POINTER(_MuRule), p]
    lib.fp8_linear_fwd.argtypes = [p, p, p, p, p, i, p, i, p, i, i, i, p]
    lib.fp8_linear_dgrad.argtypes = [p, p, p, p, p, i, p, i, i, i, p]
    lib.fp8_linear_wgrad.argtypes = [p, p, p, p, p, i, p, i, i, i, p]
    lib.fp8_adam_workspace_bytes.argtypes, lib.fp8_adam_workspace_bytes.restype = [i], sz
    for name in ("fp8_adam_step", "fp8_adam_stats", "fp8_adam_apply"):
        getattr(lib, name).argtypes = [ctypes.POINTER(_Chunk), i, ctypes.POINTER(_HParams), p, sz, p]
    lib.fp8_adam_step_noalloc.argtypes = [ctypes.POINTER(_Chunk), i, ctypes.POINTER(_HParams), p]
    lib.fp8_adam_step_into_castgrad.argtypes = [ctypes.POINTER(_Chunk), ctypes.POINTER(_Dest),
                                                ctypes.POINTER(_GradCast), i, ctypes.POINTER(_HParams), p, sz, p]
    for name in ("fp8_adam_step_into", "fp8_adam_stats_into", "fp8_adam_apply_into"):
        getattr(lib, name).argtypes = [ctypes.POINTER(_Chunk), ctypes.POINTER(_Dest), i,
                                       ctypes.POINTER(_HParams), p, sz, p]
    lib.fp8_selftest_wait_timeout.argtypes = [ctypes.c_uint, p]
    lib.fp8_selftest_step_reciprocal.argtypes = [ctypes.c_uint, ctypes.c_ulonglong, p, p, p]
    lib.fp8_selftest_encode.argtypes = [i, ctypes.c_uint, ctypes.c_ulonglong, p, p, p]
    lib.fp8_get_status.argtypes = [ctypes.POINTER(ctypes.c_uint), p]
    lib.fp8_strerror.argtypes, lib.fp8_strerror.restype = [i], ctypes.c_char_p
    for name in SYMBOLS:
        if name not in ("fp8_adam_workspace_bytes", "fp8_strerror"):
            getattr(lib, name).restype = i
    _lib = lib
    return lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libfp8 takes device tensors")
    return t.data_ptr()


def _check(rc: int, what: str) -> None:
    if rc != FP8_OK:
        raise FP8Error(rc, what)


def fp8_strerror(code: int) -> str:
    return load_library().fp8_strerror(code).decode()


# ---------------------------------------------------------------- amax / scale / cast
def fp8_amax(x: torch.Tensor, amax_out: torch.Tensor, stream=None) -> None:
    """amax_out[0] = max |x| (float32 device scalar)."""
    _check(load_library().fp8_amax(_ptr(x), _DT[x.dtype], x.numel(), _ptr(amax_out), _stream(stream)),
           "fp8_amax")


def fp8_compute_scale(amax: torch.Tensor, fmt: int, margin: int, mu: float, scale_out: torch.Tensor,
                      inv_scale_out: torch.Tensor, stream=None) -> None:
    _check(load_library().fp8_compute_scale(_ptr(amax), fmt, margin, mu, _ptr(scale_out),
                                            _ptr(inv_scale_out), _stream(stream)), "fp8_compute_scale")


def fp8_cast(x: torch.Tensor, fmt: int, scale: torch.Tensor, q_out: torch.Tensor, stream=None) -> None:
    """q_out = enc_fmt(x * scale): uint8 codes, or 16-bit halves for FP8_F16S."""
    _check(load_library().fp8_cast(_ptr(x), _DT[x.dtype], x.numel(), fmt, _ptr(scale), _ptr(q_out),
                                   _stream(stream)), "fp8_cast")


def fp8_scale_cast(x: torch.Tensor, fmt: int, amax: torch.Tensor, margin: int, mu: float,
                   scale_out: torch.Tensor, inv_scale_out: torch.Tensor, q_out: torch.Tensor,
                   stream=None) -> None:
    """fp8_compute_scale + fp8_cast in one launch."""
    _check(load_library().fp8_scale_cast(_ptr(x), _DT[x.dtype], x.numel(), fmt, _ptr(amax), margin, mu,
                                         _ptr(scale_out), _ptr(inv_scale_out), _ptr(q_out),
                                         _stream(stream)), "fp8_scale_cast")


def fp8_amax_scale_cast(x: torch.Tensor, fmt: int, amax_out: torch.Tensor, margin: int, mu: float,
                        scale: torch.Tensor, inv_scale_out: torch.Tensor, q_out: torch.Tensor,
                        stream=None) -> None:
    """fp8_amax + fp8_scale_cast in one pass over x when the scale holds:
    `scale` holds the predicted scale on entry (the tensor's previous one) and
    the new scale on return."""
    _check(load_library().fp8_amax_scale_cast(_ptr(x), _DT[x.dtype], x.numel(), fmt, _ptr(amax_out), margin, mu,
                                              _ptr(scale), _ptr(inv_scale_out), _ptr(q_out), _stream(stream)),
           "fp8_amax_scale_cast")


# ---------------------------------------------------------------- scaling variants, FP8 all-reduce
def fp8_cast_count(x: torch.Tensor, fmt: int, scale: torch.Tensor, q_out: torch.Tensor, counts: torch.Tensor,
                   stream=None) -> None:
    """fp8_cast, adding (underflows, overflows) to counts (2 x int64, device)."""
    _check(load_library().fp8_cast_count(_ptr(x), _DT[x.dtype], x.numel(), fmt, _ptr(scale), _ptr(q_out),
                                         _ptr(counts), _stream(stream)), "fp8_cast_count")


def fp8_grad_cast(g: torch.Tensor, fmt: int, amax: torch.Tensor, margin: int, mu: torch.Tensor,
                  scale_out: torch.Tensor, inv_scale_out: torch.Tensor, q_out: torch.Tensor,
                  counts: torch.Tensor | None = None, stream=None) -> None:
    """Payload cast of the FP8 gradient all-reduce: S = mu * 2^(floor(log2(fmax/amax)) - margin)."""
    _check(load_library().fp8_grad_cast(_ptr(g), _DT[g.dtype], g.numel(), fmt, _ptr(amax), margin, _ptr(mu),
                                        _ptr(scale_out), _ptr(inv_scale_out), _ptr(q_out), _ptr(counts),
                                        _stream(stream)), "fp8_grad_cast")


def fp8_sum_codes(rows: torch.Tensor, n: int, fmt: int, out: torch.Tensor, inv_scale: torch.Tensor | None = None,
                  g_inv_out: torch.Tensor | None = None, counts: torch.Tensor | None = None,
                  stream=None) -> None:
    """out[:n] = enc(sum over the rows of rows[:, :n]), rows = [nranks, ld] uint8."""
    nranks, ld = rows.shape
    _check(load_library().fp8_sum_codes(_ptr(rows), nranks, ld, n, fmt, _ptr(out), _ptr(inv_scale),
                                        _ptr(g_inv_out), _ptr(counts), _stream(stream)), "fp8_sum_codes")


def fp8_mu_update(mu: torch.Tensor, clean: torch.Tensor, counts: torch.Tensor, n: int, theta: float,
                  interval: int, mu_min: float, mu_max: float, stream=None) -> None:
    """The auto-scaling rule for mu (device state; clears counts)."""
    rule = _MuRule(theta, interval, mu_min, mu_max)
    _check(load_library().fp8_mu_update(_ptr(mu), _ptr(clean), _ptr(counts), n, ctypes.byref(rule),
                                        _stream(stream)), "fp8_mu_update")


# ---------------------------------------------------------------- GEMMs
def _out_dt(t, rto: bool) -> int:
    """Output type code; rto asks a bfloat16 output to be rounded to odd."""
    if rto:
        if t.dtype != torch.bfloat16:
            raise TypeError("a round-to-odd output is bfloat16")
        return FP8_DT_BF16_RTO
    return _DT[t.dtype]


def fp8_linear_fwd(xq, x_inv, wq, w_inv, y, y_amax=None, bias=None, stream=None, rto=False) -> None:
    """y[M,N] = (xq[M,K] . wq[N,K]^T) * x_inv * w_inv (+ bias)."""
    M, K = xq.shape
    N = wq.shape[0]
    _check(load_library().fp8_linear_fwd(_ptr(xq), _ptr(x_inv), _ptr(wq), _ptr(w_inv), _ptr(bias),
                                         _DT[bias.dtype] if bias is not None else 0, _ptr(y), _out_dt(y, rto),
                                         _ptr(y_amax), M, N, K, _stream(stream)), "fp8_linear_fwd")


def fp8_linear_dgrad(dyq, dy_inv, wq, w_inv, dx, dx_amax=None, stream=None, rto=False) -> None:
    """dx[M,K] = (dyq[M,N] . wq[N,K]) * dy_inv * w_inv."""
    M, N = dyq.shape
    K = wq.shape[1]
    _check(load_library().fp8_linear_dgrad(_ptr(dyq), _ptr(dy_inv), _ptr(wq), _ptr(w_inv), _ptr(dx),
                                           _out_dt(dx, rto), _ptr(dx_amax), M, N, K, _stream(stream)),
           "fp8_linear_dgrad")


def fp8_linear_wgrad(dyq, dy_inv, xq, x_inv, dw, dw_amax=None, stream=None, rto=False) -> None:
    """dw[N,K] = (dyq[M,N]^T . xq[M,K]) * dy_inv * x_inv.  rto: a bfloat16 dw
    rounded to odd, the form whose FP8 gradient cast gives exactly the codes
    and scale of the float32 dw's (half the bytes written and read)."""
    M, N = dyq.shape
    K = xq.shape[1]
    _check(load_library().fp8_linear_wgrad(_ptr(dyq), _ptr(dy_inv), _ptr(xq), _ptr(x_inv), _ptr(dw),
                                           _out_dt(dw, rto), _ptr(dw_amax), M, N, K, _stream(stream)),
           "fp8_linear_wgrad")


# ---------------------------------------------------------------- Adam
@dataclass
class AdamChunk:
    """Stored state of one tensor: E5M2 grad codes + g_inv, E4M3 m1 codes +
    scale, FP16 m2 bits + scale, FP16 master bits + scale (device tensors).
    Optional: w_amax (tracked amax of the stored master, -1 = unknown) and
    wq, wq_scale, wq_inv (E4M3 copy of the new master and its scales)."""
    g: torch.Tensor
    g_inv: torch.Tensor
    m: torch.Tensor
    m_scale: torch.Tensor
    v: torch.Tensor
    v_scale: torch.Tensor
    w: torch.Tensor
    w_scale: torch.Tensor
    w_amax: torch.Tensor | None = None
    wq: torch.Tensor | None = None
    wq_scale: torch.Tensor | None = None
    wq_inv: torch.Tensor | None = None


def fp8_adam_workspace_bytes(nchunks: int) -> int:
    return load_library().fp8_adam_workspace_bytes(nchunks)


def pack_adam_chunks(chunks: list[AdamChunk]):
    """Host array of fp8_adam_chunk (reusable across steps)."""
    arr = (_Chunk * len(chunks))()
    for i, c in enumerate(chunks):
        arr[i] = _Chunk(_ptr(c.g), _ptr(c.g_inv), _ptr(c.m), _ptr(c.m_scale), _ptr(c.v), _ptr(c.v_scale),
                        _ptr(c.w), _ptr(c.w_scale), c.g.numel(), _ptr(c.w_amax), _ptr(c.wq),
                        _ptr(c.wq_scale), _ptr(c.wq_inv))
    return arr


def fp8_adam_step(chunks, lr: float, beta1: float, beta2: float, eps: float, step: int, margin: int,
                  workspace: torch.Tensor, stream=None) -> None:
    """One decoupled FP8 Adam step over every chunk (in place).  `chunks` is a
    list of AdamChunk or the array returned by pack_adam_chunks."""
    arr = chunks if isinstance(chunks, ctypes.Array) else pack_adam_chunks(chunks)
    hp = _HParams(lr, beta1, beta2, eps, step, margin)
    _check(load_library().fp8_adam_step(arr, len(arr), ctypes.byref(hp), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream)),
           "fp8_adam_step")


def pack_adam_dests(dests) -> ctypes.Array:
    """Host array of fp8_adam_dest from (m, v, w) device tensors per chunk."""
    arr = (_Dest * len(dests))()
    for i, (m, v, w) in enumerate(dests):
        arr[i] = _Dest(_ptr(m), _ptr(v), _ptr(w))
    return arr


def _adam_into(name, chunks, dests, lr, beta1, beta2, eps, step, margin, workspace, stream):
    arr = chunks if isinstance(chunks, ctypes.Array) else pack_adam_chunks(chunks)
    darr = dests if isinstance(dests, ctypes.Array) else pack_adam_dests(dests)
    if len(darr) != len(arr):
        raise ValueError("one dest per chunk")
    hp = _HParams(lr, beta1, beta2, eps, step, margin)
    _check(getattr(load_library(), name)(arr, darr, len(arr), ctypes.byref(hp), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)), name)


def fp8_adam_step_into(chunks, dests, lr: float, beta1: float, beta2: float, eps: float, step: int,
                       margin: int, workspace: torch.Tensor, stream=None) -> None:
    """The step of fp8_adam_step with the new m, v, w written into `dests`
    (a list of (m, v, w) tensors per chunk, or pack_adam_dests' array); the
    chunks' own m, v, w are only read.  Bit for bit the in-place step's
    results, in one pass over the state when the scales do not change."""
    _adam_into("fp8_adam_step_into", chunks, dests, lr, beta1, beta2, eps, step, margin, workspace, stream)


def pack_grad_amax(amaxes) -> ctypes.Array:
    """Host array of the dev pointers of per-chunk gradient amaxes."""
    arr = (ctypes.c_void_p * len(amaxes))()
    for i, a in enumerate(amaxes):
        arr[i] = _ptr(a)
    return arr


def fp8_adam_step_into_castgrad(chunks, dests, grad_amax, mu: float, grad_margin: int, lr: float, beta1: float,
                                beta2: float, eps: float, step: int, margin: int, workspace: torch.Tensor,
                                stream=None) -> None:
    """fp8_adam_step_into with the gradient cast in the pass: each chunk's g is
    the bfloat16 dW (the wgrad's output), cast to E5M2 with the scale of its
    amax (grad_amax: per chunk a device scalar, or pack_grad_amax's array),
    mu and grad_margin -- the codes fp8_scale_cast would write, never
    stored; each chunk's g_inv receives the gradient's inverse scale."""
    arr = chunks if isinstance(chunks, ctypes.Array) else pack_adam_chunks(chunks)
    darr = dests if isinstance(dests, ctypes.Array) else pack_adam_dests(dests)
    amax = grad_amax if isinstance(grad_amax, ctypes.Array) else pack_grad_amax(grad_amax)
    if len(darr) != len(arr) or len(amax) != len(arr):
        raise ValueError("one dest and one gradient amax per chunk")
    gc = _GradCast(ctypes.cast(amax, ctypes.POINTER(ctypes.c_void_p)), mu, grad_margin)
    hp = _HParams(lr, beta1, beta2, eps, step, margin)
    _check(load_library().fp8_adam_step_into_castgrad(arr, darr, ctypes.byref(gc), len(arr), ctypes.byref(hp),
                                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                      _stream(stream)), "fp8_adam_step_into_castgrad")


def fp8_adam_stats_into(chunks, dests, lr: float, beta1: float, beta2: float, eps: float, step: int,
                        margin: int, workspace: torch.Tensor, stream=None) -> None:
    """First half of the element-sharded out-of-place step: this rank's new
    slices into `dests` with the predicted scales, the exact new amaxes into
    `workspace` (to be MAX-reduced over the ranks)."""
    _adam_into("fp8_adam_stats_into", chunks, dests, lr, beta1, beta2, eps, step, margin, workspace, stream)


def fp8_adam_apply_into(chunks, dests, lr: float, beta1: float, beta2: float, eps: float, step: int,
                        margin: int, workspace: torch.Tensor, stream=None) -> None:
    """Second half: the new scales from the reduced workspace, and the slices
    of the tensors whose scales changed written again."""
    _adam_into("fp8_adam_apply_into", chunks, dests, lr, beta1, beta2, eps, step, margin, workspace, stream)


def _adam_half(name, chunks, lr, beta1, beta2, eps, step, margin, workspace, stream):
    arr = chunks if isinstance(chunks, ctypes.Array) else pack_adam_chunks(chunks)
    hp = _HParams(lr, beta1, beta2, eps, step, margin)
    _check(getattr(load_library(), name)(arr, len(arr), ctypes.byref(hp), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)), name)


def fp8_adam_stats(chunks, lr: float, beta1: float, beta2: float, eps: float, step: int, margin: int,
                   workspace: torch.Tensor, stream=None) -> None:
    """First half of an element-sharded step: amax of this rank's new m, v, w
    per chunk into `workspace` (state unchanged)."""
    _adam_half("fp8_adam_stats", chunks, lr, beta1, beta2, eps, step, margin, workspace, stream)


def fp8_adam_apply(chunks, lr: float, beta1: float, beta2: float, eps: float, step: int, margin: int,
                   workspace: torch.Tensor, stream=None) -> None:
    """Second half: new scales from the (rank-reduced) workspace, then the
    in-place update of this rank's slices."""
    _adam_half("fp8_adam_apply", chunks, lr, beta1, beta2, eps, step, margin, workspace, stream)


FP8_ADAM_NOALLOC_MAX_CHUNKS = 1024


def fp8_adam_step_noalloc(chunks, lr: float, beta1: float, beta2: float, eps: float, step: int,
                          margin: int, stream=None) -> None:
    """fp8_adam_step for callers that cannot provide device memory: the
    library's fixed per-device scratch array replaces the workspace (at most
    FP8_ADAM_NOALLOC_MAX_CHUNKS chunks; calls overlapping on the GPU race)."""
    arr = chunks if isinstance(chunks, ctypes.Array) else pack_adam_chunks(chunks)
    hp = _HParams(lr, beta1, beta2, eps, step, margin)
    _check(load_library().fp8_adam_step_noalloc(arr, len(arr), ctypes.byref(hp), _stream(stream)),
           "fp8_adam_step_noalloc")


def fp8_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Run the GEMM pipeline's bounded wait on a barrier nothing arrives at
    (limit in microseconds); it must end and raise FP8_STATUS_TIMEOUT."""
    _check(load_library().fp8_selftest_wait_timeout(ctypes.c_uint(limit_us), _stream(stream)),
           "fp8_selftest_wait_timeout")


def fp8_selftest_step_reciprocal(lo_bits: int, hi_bits: int, bad: torch.Tensor, first: torch.Tensor,
                                 stream=None) -> None:
    """Compare the Adam step's reciprocal with CUDA's correctly rounded one on
    the binary32 bit patterns [lo_bits, hi_bits); bad (1 x int64) counts
    differences, first (1 x int32) gets the smallest differing pattern (both
    initialised by the caller)."""
    _check(load_library().fp8_selftest_step_reciprocal(lo_bits, hi_bits, _ptr(bad), _ptr(first),
                                                       _stream(stream)), "fp8_selftest_step_reciprocal")


def fp8_selftest_encode(fmt: int, lo_bits: int, hi_bits: int, bad: torch.Tensor, first: torch.Tensor,
                        stream=None) -> None:
    """Compare the library's branch-free FP8 encoder with the explicitly
    checked one on the binary32 bit patterns [lo_bits, hi_bits), in both
    lanes; bad (1 x int64) counts differences, first (1 x int32) gets the
    smallest differing pattern (both initialised by the caller)."""
    _check(load_library().fp8_selftest_encode(fmt, lo_bits, hi_bits, _ptr(bad), _ptr(first), _stream(stream)),
           "fp8_selftest_encode")


def fp8_get_status(stream=None) -> int:
    """Wait for the stream, read and clear the device status word."""
    out = ctypes.c_uint(0)
    _check(load_library().fp8_get_status(ctypes.byref(out), _stream(stream)), "fp8_get_status")
    return out.value
