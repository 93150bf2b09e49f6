"""The allocation-free Adam entry point against the workspace one.

Some callers cannot give the library any device memory: code inside a host
framework whose caching allocator already owns the GPU's memory, plugins
whose host forbids raw cudaMalloc, and loops that must never take the
device-wide synchronisation that cudaMalloc/cudaFree can cause.
fp8_adam_step_noalloc serves them from a fixed scratch array inside the
library.  It runs the same kernels with the same arithmetic as fp8_adam_step,
so through the C ABI two consecutive calls must leave bit for bit the same
state: codes, FP16 values and scales.  One case has more than 224 chunks, so
the step runs as two launch groups that use different parts of the scratch
array.

This file is collected last on purpose, and it also passes alone in a fresh
process (the scratch array is set up on the first call).
"""
import numpy as np
import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8
from test_gpu_parity import HP, make_adam_state, snapshot

pytestmark = pytest.mark.gpu


def _assert_identical(got, ref, what):
    for k in ("m", "v", "w", "s_m", "s_v", "s_w"):
        assert np.array_equal(np.asarray(got[k]), np.asarray(ref[k])), (what, k)


@pytest.mark.parametrize("sizes", [[65536, 4099, 7, 300000], [37 + 16 * i for i in range(300)]],
                         ids=["4-chunks", "300-chunks"])
def test_noalloc_matches_workspace_step_on_two_calls(sizes):
    assert len(sizes) <= fp8.FP8_ADAM_NOALLOC_MAX_CHUNKS
    ref = make_adam_state(sizes, ("noalloc", len(sizes)))
    new = make_adam_state(sizes, ("noalloc", len(sizes)))
    for i, (r, n) in enumerate(zip(ref, new)):  # identical starting states
        _assert_identical(snapshot(n), snapshot(r), ("start", i))
    ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(ref)) // 4, dtype=torch.float32, device="cuda")
    for step in (1, 2):
        fp8.fp8_adam_step(ref, step=step, margin=0, workspace=ws, **HP)
        fp8.fp8_adam_step_noalloc(new, step=step, margin=0, **HP)
        assert fp8.fp8_get_status() == 0
        for i, (r, n) in enumerate(zip(ref, new)):
            _assert_identical(snapshot(n), snapshot(r), (step, i))


def test_noalloc_rejects_more_chunks_than_its_scratch_holds():
    chunks = make_adam_state([16], ("noalloc-limit",)) * (fp8.FP8_ADAM_NOALLOC_MAX_CHUNKS + 1)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_adam_step_noalloc(chunks, step=1, margin=0, **HP)
    assert e.value.code == fp8.FP8_ERR_INVALID_ARG
