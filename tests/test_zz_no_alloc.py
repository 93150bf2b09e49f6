"""The allocation-free Adam entry point against the workspace one.

Some callers cannot give the library any device memory: code inside a host
framework whose caching allocator already owns the GPU's memory, plugins
whose host forbids raw cudaMalloc, and loops that must never take the
device-wide synchronisation that cudaMalloc/cudaFree can cause.
fp8_adam_step_noalloc serves them from a fixed scratch array inside the
library.  Through the C ABI, two consecutive calls must leave the same state
as fp8_adam_step within the parity tolerances: scales equal, master weights
and second moment within 1 FP16 ULP, first-moment codes within 1 code.

This file is collected last on purpose, and it also passes alone in a fresh
process (the scratch array is set up on the first call).
"""
import numpy as np
import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8
from _util import code_rank, f16_ulp, f16_vals
from test_gpu_parity import HP, make_adam_state, snapshot

pytestmark = pytest.mark.gpu

SIZES = [65536, 4099, 7, 300000]


def _assert_same_state(got, ref):
    assert (got["s_m"], got["s_v"], got["s_w"]) == (ref["s_m"], ref["s_v"], ref["s_w"])
    for key, skey in (("w", "s_w"), ("v", "s_v")):
        a = f16_vals(got[key]) / got[skey]
        b = f16_vals(ref[key]) / ref[skey]
        assert np.all(np.abs(a - b) <= f16_ulp(f16_vals(ref[key])) / ref[skey]), key
    assert np.all(np.abs(code_rank(got["m"]) - code_rank(ref["m"])) <= 1)


def test_noalloc_matches_workspace_step_on_two_calls():
    ref = make_adam_state(SIZES, ("noalloc",))
    new = make_adam_state(SIZES, ("noalloc",))
    for r, n in zip(ref, new):  # identical starting states
        sr, sn = snapshot(r), snapshot(n)
        assert all(np.array_equal(np.asarray(sr[k]), np.asarray(sn[k])) for k in sr)
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(ref)) // 4, dtype=torch.float32, device="cuda")
    for step in (1, 2):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        fp8.fp8_adam_step_noalloc(new, step=step, margin=0, **HP)
        assert fp8.fp8_get_status() == 0
        for r, n in zip(ref, new):
            _assert_same_state(snapshot(n), snapshot(r))


def test_noalloc_rejects_more_chunks_than_its_scratch_holds():
    chunks = make_adam_state([16], ("noalloc-limit",)) * (fp8.FP8_ADAM_NOALLOC_MAX_CHUNKS + 1)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_adam_step_noalloc(chunks, step=1, margin=0, **HP)
    assert e.value.code == fp8.FP8_ERR_INVALID_ARG
