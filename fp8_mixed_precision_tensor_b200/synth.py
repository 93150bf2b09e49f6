"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and nothing else: it holds none of the FP8
method's arithmetic (no scaling, casting, GEMM or optimizer math), so the same
seeded bytes can feed the CUDA path and any independent CPU checker.  Host arrays come from numpy
PCG64 generators keyed by (workload, tensor, step); large device-resident
benchmark inputs come from torch's seeded CUDA generator with the same value
distributions.  fp32 -> bf16 input rounding is round-to-nearest-even.

Workload shapes follow the pages' models: GPT-7B (hidden 4096, 32 layers) and
GPT-175B (hidden 12288) from "FP8-LM: Training FP8 Large Language Models",
実験設定, and GPT/Llama-2 7B-70B from "Training and inference of large
language models using 8-bit floating point".
"""
from __future__ import annotations

import zlib

import numpy as np


def key_seed(*key) -> int:
    """Stable 32-bit seed from a tuple of names/ints (crc32 of its repr)."""
    return zlib.crc32(repr(tuple(key)).encode())


def rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(key_seed(*key)))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (input preparation)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_f32(shape, std: float, *key) -> np.ndarray:
    return (rng(*key).standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def normal_bf16(shape, std: float, *key) -> np.ndarray:
    return to_bf16_bits(normal_f32(shape, std, *key))


def lognormal_outliers_bf16(n: int, *key) -> np.ndarray:
    """sign * exp(N(-3, 2)), Bernoulli(1/2) sign; 0.01 % of the indices
    (without replacement) multiplied by 1e3; then 0.1 % set to exactly +0
    (zeros are applied last).  Returned as bf16 bits."""
    g = rng(*key)
    x = np.exp(g.normal(-3.0, 2.0, n)).astype(np.float32)
    x *= np.where(g.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
    n_out = max(1, n // 10000)
    x[g.choice(n, n_out, replace=False)] *= np.float32(1e3)
    n_zero = max(1, n // 1000)
    x[g.choice(n, n_zero, replace=False)] = 0.0
    return to_bf16_bits(x)


# ---------------------------------------------------------------- workloads
SINGLE_LINEAR_256 = dict(M=256, N=256, K=256, x_std=1.0, w_std=0.02, dy_std=1e-4)

# GPT-7B transformer-block linears, tokens = batch 2 x seq 2048, hidden 4096.
GPT7B_LINEARS = [  # (name, K in, N out)
    ("qkv", 4096, 12288),
    ("out_proj", 4096, 4096),
    ("fc1", 4096, 16384),
    ("fc2", 16384, 4096),
]
GPT7B_TOKENS = 4096
GPT7B_W_STD = 0.02

# GPT-175B transformer-block linears, tokens = batch 4 x seq 2048, hidden 12288.
GPT175B_LINEARS = [
    ("qkv", 12288, 36864),
    ("out_proj", 12288, 12288),
    ("fc1", 12288, 49152),
    ("fc2", 49152, 12288),
]
GPT175B_TOKENS = 8192
GPT175B_W_STD = 0.006

ACT_STD = 1.0
GRAD_STD = 1e-4


def gpt7b_adam_chunks() -> list[tuple[str, int]]:
    """Per-tensor parameter chunks of GPT-7B: 32 layers x (QKV, out, fc1, fc2)
    plus the 50304 x 4096 embedding (LayerNorm/bias vectors omitted)."""
    chunks = []
    for layer in range(32):
        for name, k, n in GPT7B_LINEARS:
            chunks.append((f"l{layer}.{name}", k * n))
    chunks.append(("embedding", 50304 * 4096))
    return chunks


def linear_inputs_f32(M: int, N: int, K: int, x_std: float, w_std: float, dy_std: float, *key):
    """X[M,K], W[N,K], dY[M,N] as fp32 arrays."""
    return (normal_f32((M, K), x_std, *key, "X"), normal_f32((N, K), w_std, *key, "W"),
            normal_f32((M, N), dy_std, *key, "dY"))


def linear_inputs_bf16(M: int, N: int, K: int, x_std: float, w_std: float, dy_std: float, *key):
    """X[M,K], W[N,K], dY[M,N] as bf16 bit arrays."""
    return tuple(to_bf16_bits(a) for a in linear_inputs_f32(M, N, K, x_std, w_std, dy_std, *key))


def adam_grad_f32(n: int, std: float, *key) -> np.ndarray:
    return normal_f32((n,), std, *key)


# ---------------------------------------------------------------- device-side (large)
def device_normal(shape, std: float, seed: int, dtype, device):
    """Seeded N(0, std) tensor generated directly in device memory (for
    benchmark inputs too large to draw on the host)."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=gen)
    return t.to(dtype)
