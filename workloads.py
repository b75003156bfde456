"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and shapes them into the workloads below. It holds
none of the quantization or attention arithmetic: the CUDA path and the oracle each receive
the same arrays from here and compute independently.

Workloads (d = 128 throughout):

  score      4096 fp32 keys, i.i.d. N(0,1) coordinates times a per-row scale U[2,20];
             8 fp32 N(0,1) queries; keys 3-bit prod (2-bit MSE + 1-bit QJL), quantizer seed 0.
  decode-s   batch 1, 12 query heads on 2 KV heads, context 32768; bf16 keys N(0,1) x U[2,20]
             per row, bf16 N(0,1) values, one bf16 N(0,1) query token; keys 3-bit prod,
             values 2-bit groups of 32.
  decode-l   batch 8, 28 query heads on 4 KV heads, context 32768; as decode-s plus, per
             (sequence, KV head), 16 planted keys 0.9*q + 0.1*N(0,1) where q is the first
             query head of that KV group.
  quantize   2^24 bf16 rows = 4 layers x 2^22 rows; N(0,1) with 32 fixed channels at 4x std;
             quantizer seed = layer index.
  stream     batch 1, 64 query heads on 8 KV heads, context 131072 bf16 (distributed as
             decode-s); keys 4-bit prod, values 4-bit groups of 32; 256 steps of
             append(1 token per KV head) + decode.

Data seed = workload number (1..5). bf16 inputs are rounded from fp32 draws with
round-to-nearest-even (torch's conversion) and handed to both sides as those exact values.
"""
from __future__ import annotations

import numpy as np

D = 128

WORKLOADS = {
    1: dict(name="score", n_keys=4096, n_queries=8, mode="prod", key_bits=3, qseed=0,
            dtype="f32"),
    2: dict(name="decode-s", batch=1, n_q_heads=12, n_kv_heads=2, ctx=32768, mode="prod",
            key_bits=3, value_bits=2, group=32, qseed=0, dtype="bf16"),
    3: dict(name="decode-l", batch=8, n_q_heads=28, n_kv_heads=4, ctx=32768, mode="prod",
            key_bits=3, value_bits=2, group=32, qseed=0, dtype="bf16", planted=16),
    4: dict(name="quantize", rows=1 << 24, layers=4, n_outlier=32, outlier_std=4.0,
            dtype="bf16"),
    5: dict(name="stream", batch=1, n_q_heads=64, n_kv_heads=8, ctx=131072, steps=256,
            mode="prod", key_bits=4, value_bits=4, group=32, qseed=0, dtype="bf16"),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to bf16 (RNE) and returned as fp32 (exactly representable)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def scaled_gaussian_rows(g: np.random.Generator, n: int, d: int = D,
                         lo: float = 2.0, hi: float = 20.0) -> np.ndarray:
    """n rows of i.i.d. N(0,1) coordinates, each row multiplied by its own U[lo, hi] scale."""
    x = g.standard_normal((n, d), dtype=np.float32)
    s = g.uniform(lo, hi, size=(n, 1)).astype(np.float32)
    return x * s


def gaussian(g: np.random.Generator, shape) -> np.ndarray:
    return g.standard_normal(shape, dtype=np.float32)


def outlier_channels(seed: int, d: int = D, n_out: int = 32) -> np.ndarray:
    """The fixed high-variance channels of the quantize workload (sorted)."""
    return np.sort(rng(seed).choice(d, n_out, replace=False)).astype(np.int32)


def outlier_rows(g: np.random.Generator, n: int, channels: np.ndarray, d: int = D,
                 boost: float = 4.0) -> np.ndarray:
    x = g.standard_normal((n, d), dtype=np.float32)
    x[:, channels] *= np.float32(boost)
    return x


def score_inputs(seed: int = 1, n_keys: int = 4096, n_queries: int = 8):
    """Keys (fp32, n_keys x 128) and queries (fp32, n_queries x 128) of the score workload."""
    g = rng(seed)
    keys = scaled_gaussian_rows(g, n_keys)
    queries = gaussian(g, (n_queries, D))
    return keys, queries


def decode_inputs(seed: int, batch: int, n_q_heads: int, n_kv_heads: int, ctx: int,
                  planted: int = 0, extra_tokens: int = 0):
    """K, V as bf16-exact fp32 arrays of shape (batch, n_kv_heads, ctx + extra_tokens, 128),
    q as (batch, n_q_heads, 128), and the planted positions (batch, n_kv_heads, planted).

    extra_tokens rows are appended after the context (fresh tokens for streaming append)."""
    g = rng(seed)
    n = ctx + extra_tokens
    k = scaled_gaussian_rows(g, batch * n_kv_heads * n).reshape(batch, n_kv_heads, n, D)
    v = gaussian(g, (batch, n_kv_heads, n, D))
    q = gaussian(g, (batch, n_q_heads, D))
    q = round_bf16(q)
    pos = np.zeros((batch, n_kv_heads, planted), dtype=np.int64)
    if planted:
        group = n_q_heads // n_kv_heads
        for b in range(batch):
            for h in range(n_kv_heads):
                p = np.sort(g.choice(ctx, planted, replace=False))
                pos[b, h] = p
                noise = gaussian(g, (planted, D))
                k[b, h, p] = np.float32(0.9) * q[b, h * group][None, :] + np.float32(0.1) * noise
    return round_bf16(k), round_bf16(v), q, pos


def quantize_rows_numpy(seed: int, n: int, channels: np.ndarray) -> np.ndarray:
    """bf16-exact rows of the quantize workload, generated on the host (small n only)."""
    return round_bf16(outlier_rows(rng(seed), n, channels))
