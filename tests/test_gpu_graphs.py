"""The library's calls captured in a CUDA graph (stream capture) and replayed
give exactly what the same calls give when issued one by one: the scale and
cast chain, the three GEMMs with their fused amaxes, the gradient cast and
the Adam step.  Small tensors are launch-bound when issued from Python; a
graph is how a caller removes that host cost."""
import numpy as np
import pytest
import torch

from fp8_mixed_precision_tensor_b200 import fp8, synth
from test_gpu_parity import HP, make_adam_state, snapshot

pytestmark = pytest.mark.gpu

F32 = dict(dtype=torch.float32, device="cuda")


def _linear_buffers(M, N, K):
    X = synth.device_normal((M, K), 1.0, 21, torch.bfloat16, "cuda")
    W = synth.device_normal((N, K), 0.02, 22, torch.bfloat16, "cuda")
    dY = synth.device_normal((M, N), 1e-4, 23, torch.bfloat16, "cuda")
    u8 = dict(dtype=torch.uint8, device="cuda")
    return dict(X=X, W=W, dY=dY, xq=torch.empty((M, K), **u8), wq=torch.empty((N, K), **u8),
                dyq=torch.empty((M, N), **u8), y=torch.empty((M, N), dtype=torch.bfloat16, device="cuda"),
                dx=torch.empty((M, K), dtype=torch.bfloat16, device="cuda"), dw=torch.empty((N, K), **F32),
                gq=torch.empty((N, K), **u8), sc=torch.zeros(16, **F32))


def _linear_pass(b):
    sc = b["sc"]
    for t, q, i, fmt, mu in ((b["X"], b["xq"], 0, fp8.FP8_E4M3, 1.0), (b["W"], b["wq"], 3, fp8.FP8_E4M3, 1.0),
                             (b["dY"], b["dyq"], 6, fp8.FP8_E5M2, 2.0 ** 10)):
        fp8.fp8_amax(t, sc[i:i + 1])
        fp8.fp8_scale_cast(t, fmt, sc[i:i + 1], 0, mu, sc[i + 1:i + 2], sc[i + 2:i + 3], q)
    fp8.fp8_linear_fwd(b["xq"], sc[2:3], b["wq"], sc[5:6], b["y"], sc[12:13])
    fp8.fp8_linear_dgrad(b["dyq"], sc[8:9], b["wq"], sc[5:6], b["dx"], sc[13:14])
    fp8.fp8_linear_wgrad(b["dyq"], sc[8:9], b["xq"], sc[2:3], b["dw"], sc[14:15])
    fp8.fp8_scale_cast(b["dw"], fp8.FP8_E5M2, sc[14:15], 0, 2.0 ** 10, sc[10:11], sc[11:12], b["gq"])


@pytest.mark.parametrize("shape", [(512, 1024, 512), (2320, 4624, 528)])
def test_linear_pass_in_a_cuda_graph_equals_eager(shape):
    M, N, K = shape
    eager, graphed = _linear_buffers(M, N, K), _linear_buffers(M, N, K)
    _linear_pass(eager)
    _linear_pass(graphed)  # first call outside the capture (device set-up)
    for k in ("xq", "wq", "dyq", "y", "dx", "dw", "gq", "sc"):
        graphed[k].zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _linear_pass(graphed)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert fp8.fp8_get_status() == 0
    for k in ("xq", "wq", "dyq", "y", "dx", "dw", "gq", "sc"):
        assert torch.equal(eager[k], graphed[k]), k


def test_adam_step_in_a_cuda_graph_equals_eager():
    sizes = [65536 + 5, 4099]
    eager = make_adam_state(sizes, ("graph-adam",))
    graphed = make_adam_state(sizes, ("graph-adam",))
    ws_e = torch.zeros(fp8.fp8_adam_workspace_bytes(2) // 4, **F32)
    ws_g = torch.zeros_like(ws_e)
    arr = fp8.pack_adam_chunks(graphed)
    fp8.fp8_adam_step(eager, step=1, margin=0, workspace=ws_e, **HP)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fp8.fp8_adam_step(arr, step=1, margin=0, workspace=ws_g, **HP)
    g.replay()
    torch.cuda.synchronize()
    assert fp8.fp8_get_status() == 0
    for a, b in zip(eager, graphed):
        sa, sb = snapshot(a), snapshot(b)
        for k in ("m", "v", "w", "s_m", "s_v", "s_w"):
            assert np.array_equal(np.asarray(sa[k]), np.asarray(sb[k])), k

