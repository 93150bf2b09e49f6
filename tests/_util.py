"""Helpers shared by the GPU parity tests (comparison rules, device copies)."""
import numpy as np
import torch

# GEMM tolerance: |gpu - oracle| <= 1e-3 * sum_k |a_ik b_kj| (plus half an ULP
# of a 16-bit output type for the final rounding).
GEMM_REL = 1e-3


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.view(dtype)


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return to_dev(bits.view(np.int16)).view(torch.bfloat16)


def code_rank(c: np.ndarray) -> np.ndarray:
    """Monotone integer order of FP8 codes (-0 and +0 share rank 0)."""
    c = np.asarray(c).astype(np.int64)
    return np.where(c < 128, c, 128 - c)


def f16_vals(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits).view(np.uint16).view(np.float16).astype(np.float64)


def f16_ulp(vals: np.ndarray) -> np.ndarray:
    """Unit in the last place of binary16 values: 2^(e - 10) in the binade
    [2^e, 2^(e+1)), 2^-24 among subnormals, 32 at the largest finite 65504
    (np.spacing would step past it to inf)."""
    a = np.abs(np.asarray(vals)).astype(np.float16).astype(np.float64)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def half_ulp_out(ref: np.ndarray, out_dtype: torch.dtype) -> np.ndarray:
    if out_dtype == torch.float32:
        return np.zeros_like(ref)
    if out_dtype == torch.float16:
        return 0.5 * f16_ulp(ref)
    # bf16: 8 significant bits
    e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-300)))
    return 0.5 * 2.0 ** (e - 7)


def assert_gemm_close(gpu: np.ndarray, ref: np.ndarray, rabs: np.ndarray, out_dtype, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = GEMM_REL * rabs + half_ulp_out(ref, out_dtype)
    bad = err > bound
    if np.any(bad):
        i = np.argmax(err - bound)
        raise AssertionError(f"{what}: {np.count_nonzero(bad)} outputs outside tolerance; worst at flat {i}: "
                             f"gpu {gpu.flat[i]!r} oracle {ref.flat[i]!r} bound {bound.flat[i]!r}")


def tensor_to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def boundary_samples(rows: int, cols: int, n_random: int, key, tile_r=(128, 256), tile_c=(256,)):
    """(row, col) sample positions: random ones plus every corner and the
    first/last row and column of each tile edge (ragged edges included)."""
    from fp8_mixed_precision_tensor_b200 import synth

    g = synth.rng("samples", *key)
    r = list(g.integers(0, rows, n_random))
    c = list(g.integers(0, cols, n_random))
    edge_r = sorted({x for t in tile_r for k in range(0, rows, t) for x in (k, min(k + t, rows) - 1)})
    edge_c = sorted({x for t in tile_c for k in range(0, cols, t) for x in (k, min(k + t, cols) - 1)})
    for er in edge_r:
        for ec in g.choice(cols, min(cols, 8), replace=False).tolist() + [0, cols - 1]:
            r.append(er)
            c.append(ec)
    for ec in edge_c:
        for er in g.choice(rows, min(rows, 8), replace=False).tolist() + [0, rows - 1]:
            r.append(er)
            c.append(ec)
    return np.asarray(r, dtype=np.int64), np.asarray(c, dtype=np.int64)


def assert_codes_equal(got: np.ndarray, ref: np.ndarray, inputs=None, what=""):
    """Bit-exact comparison of code arrays; on failure the first mismatches
    with their inputs (bit patterns) are in the message."""
    got, ref = np.asarray(got).reshape(-1), np.asarray(ref).reshape(-1)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = np.nonzero(got != ref)[0]
    if bad.size:
        rows = []
        for i in bad[:8]:
            x = "" if inputs is None else f" input {np.asarray(inputs).reshape(-1)[i]!r}"
            rows.append(f"[{i}] gpu {int(got[i]):#x} oracle {int(ref[i]):#x}{x}")
        raise AssertionError(f"{what}: {bad.size} of {got.size} codes differ; " + "; ".join(rows))
