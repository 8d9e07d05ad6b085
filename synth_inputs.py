"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no retention arithmetic: it draws Gaussian tensors from a seeded
torch CPU generator, rounds them to the requested dtype (round-to-nearest-even for
bf16), and builds the per-head decay and rotary-frequency parameter arrays that both
the CUDA path and the oracle receive as inputs.

Parameter schedules (inputs to the operator, as the workloads state them):
  gamma_i = 1 - 2^(-5-i), i = 0..h-1   ("阅读笔记：RetNet", §三.2 MSR)
  theta_j = 10000^(-2j/d_k), j = 0..d_k/2-1
Both are rounded to fp32, the precision the C interface takes them in, and the
oracle upcasts those exact fp32 values.
"""
import numpy as np
import torch


def gamma_schedule(heads: int) -> np.ndarray:
    """Per-head decay 1 - 2^(-5-i) as fp32 (exact in fp32 for i <= 19; rounded above)."""
    return np.array([1.0 - 2.0 ** (-5 - i) for i in range(heads)], dtype=np.float32)


def theta_schedule(d_k: int, base: float = 10000.0) -> np.ndarray:
    """Rotary frequencies base^(-2j/d_k), one per interleaved pair, as fp32."""
    return np.array([base ** (-2.0 * j / d_k) for j in range(max(d_k // 2, 1))], dtype=np.float32)


_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def randn(shape, seed: int, dtype: str = "bf16", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) tensor on the CPU from a seeded generator, rounded to ``dtype``."""
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(_DT[dtype])


def qkv(batch, seqlen, heads, d_k, d_v, seed, dtype="bf16"):
    """Q, K: (batch, L, heads, d_k); V: (batch, L, heads, d_v), each from its own sub-seed."""
    q = randn((batch, seqlen, heads, d_k), seed * 1000 + 1, dtype)
    k = randn((batch, seqlen, heads, d_k), seed * 1000 + 2, dtype)
    v = randn((batch, seqlen, heads, d_v), seed * 1000 + 3, dtype)
    return q, k, v


def gate(batch, seqlen, heads, d_v, seed, dtype="bf16"):
    """G: (batch, L, heads*d_v), the gate input of the MSR epilogue."""
    return randn((batch, seqlen, heads * d_v), seed * 1000 + 4, dtype)


def decode_state(batch, heads, d_k, d_v, seed, std=0.01):
    """fp32 recurrent state (batch, heads, d_k, d_v) drawn as std * N(0, 1)."""
    return randn((batch, heads, d_k, d_v), seed * 1000 + 5, "f32", std=std)


def decode_token(batch, heads, d_k, d_v, seed, step, dtype="bf16"):
    """One decode step's q, k: (batch, heads, d_k) and v: (batch, heads, d_v)."""
    s = (seed * 1000 + step) * 10
    return (randn((batch, heads, d_k), s + 1, dtype), randn((batch, heads, d_k), s + 2, dtype),
            randn((batch, heads, d_v), s + 3, dtype))
