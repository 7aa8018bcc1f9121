"""Seeded synthetic inputs for the online Hadamard rotation path.

This module is shared by the tests, the benchmark and the smoke check. It
holds input synthesis only -- no step of the rotation or quantisation method
-- so that neither the CUDA path nor the CPU oracle owns the inputs both of
them are given.

Every generator draws from ``numpy.random.Generator(PCG64(seed))`` in a fixed
order, works in float32 and rounds to bfloat16 once at the end (round to
nearest even, through torch's CPU conversion). Arrays are returned as uint16
bit patterns.

Recipes (shapes and value statistics of the workloads the pages describe:
fewer than 0.1 % of channels at 100-200x the typical magnitude, outliers in
the SwiGLU product feeding the down projection):

* ``tiny``      -- 64 x 256, N(0,1), channel 7 set to 60.0.
* ``r4_prefill`` -- tokens x n, X = silu(A) * B with A, B ~ N(0,1) rounded to
  bf16 first; a seeded 0.1 % of channels multiplied by 100; seeded +-1
  diagonal as a bitmask.
* ``r3_kv``     -- Q [B,S,hq,d], K/V [B,S,hkv,d] ~ N(0,1); per head two seeded
  dims (fixed across tokens) multiplied by 50, drawn independently for Q, K
  and V; positions 0..S-1.
* ``decode``    -- tokens x n Student-t (nu = 3) = Z / sqrt(chi2_3 / 3); one
  random channel per row multiplied by 200.
* ``sweep``     -- tokens x n ~ N(0,1), max(1, round(0.001 n)) channels x 100.
"""
from __future__ import annotations

import numpy as np
import torch


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def sign_bits(n: int, seed: int) -> np.ndarray:
    """Seeded +-1 diagonal as a bitmask of n/32 uint32 words (bit j set: d_j = -1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    bits = rng.integers(0, 2, size=n, dtype=np.uint8)
    words = np.zeros((n + 31) // 32, dtype=np.uint32)
    for j in np.nonzero(bits)[0]:
        words[j >> 5] |= np.uint32(1) << np.uint32(j & 31)
    return words


def sign_vector(words: np.ndarray, n: int) -> np.ndarray:
    """Expand a sign bitmask to a +-1 float64 vector (host-side convenience)."""
    j = np.arange(n)
    bit = (np.asarray(words, dtype=np.uint32)[j >> 5] >> (j & 31).astype(np.uint32)) & 1
    return np.where(bit == 1, -1.0, 1.0)


def outlier_count(n: int) -> int:
    return max(1, int(round(0.001 * n)))


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def tiny(seed: int = 0, tokens: int = 64, n: int = 256, outlier_channel: int = 7,
         outlier_value: float = 60.0) -> np.ndarray:
    rng = _rng(seed)
    x = rng.standard_normal((tokens, n), dtype=np.float32)
    x[:, outlier_channel] = outlier_value
    return to_bf16_bits(x)


def r4_prefill(tokens: int = 8192, n: int = 16384, seed: int = 1, sign_seed: int = 101,
               block: int = 1024):
    """SwiGLU-like down-projection input. Returns (x_bits [tokens, n], signs, channels)."""
    rng = _rng(seed)
    channels = np.sort(rng.choice(n, size=outlier_count(n), replace=False))
    out = np.empty((tokens, n), dtype=np.uint16)
    for t0 in range(0, tokens, block):
        t1 = min(tokens, t0 + block)
        a = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((t1 - t0, n), dtype=np.float32)))
        b = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((t1 - t0, n), dtype=np.float32)))
        x = (a / (np.float32(1.0) + np.exp(-a))) * b
        x[:, channels] *= np.float32(100.0)
        out[t0:t1] = to_bf16_bits(x)
    return out, sign_bits(n, sign_seed), channels


def r3_kv(batch: int = 4, seq: int = 4096, n_q_heads: int = 32, n_kv_heads: int = 8,
          head_dim: int = 128, seed: int = 2):
    """Attention-shaped Q, K, V. Returns (q, k, v, pos) with bf16 bit patterns."""
    rng = _rng(seed)
    outs = []
    for heads in (n_q_heads, n_kv_heads, n_kv_heads):
        dims = np.stack([rng.choice(head_dim, size=2, replace=False) for _ in range(heads)])
        x = rng.standard_normal((batch, seq, heads, head_dim), dtype=np.float32)
        for h in range(heads):
            x[:, :, h, dims[h]] *= np.float32(50.0)
        outs.append(to_bf16_bits(x))
    pos = np.broadcast_to(np.arange(seq, dtype=np.int32), (batch, seq)).copy()
    return outs[0], outs[1], outs[2], pos


def decode(tokens: int = 32, n: int = 4096, seed: int = 3) -> np.ndarray:
    rng = _rng(seed)
    z = rng.standard_normal((tokens, n))
    chi2 = rng.chisquare(3, size=(tokens, n))
    x = (z / np.sqrt(chi2 / 3.0)).astype(np.float32)
    ch = rng.integers(0, n, size=tokens)
    x[np.arange(tokens), ch] *= np.float32(200.0)
    return to_bf16_bits(x)


def sweep(k: int, tokens: int | None = None, seed: int | None = None, block_elems: int = 1 << 26):
    """n = 2^k; default token count makes the bf16 input exactly 1 GiB."""
    n = 1 << k
    if tokens is None:
        tokens = (1 << 29) // n
    rng = _rng(4 + k if seed is None else seed)
    channels = np.sort(rng.choice(n, size=outlier_count(n), replace=False))
    out = np.empty((tokens, n), dtype=np.uint16)
    block = max(1, block_elems // n)
    for t0 in range(0, tokens, block):
        t1 = min(tokens, t0 + block)
        x = rng.standard_normal((t1 - t0, n), dtype=np.float32)
        x[:, channels] *= np.float32(100.0)
        out[t0:t1] = to_bf16_bits(x)
    return out


def weights(n_out: int = 4096, k: int = 14336, seed: int = 7, block_rows: int = 512) -> np.ndarray:
    """A linear layer's weight rows [n_out, k] as bf16 bits: N(0, 1/k) (random-init scale),
    drawn in blocks of rows from the seeded generator."""
    rng = _rng(seed)
    out = np.empty((n_out, k), dtype=np.uint16)
    for r0 in range(0, n_out, block_rows):
        r1 = min(n_out, r0 + block_rows)
        w = rng.standard_normal((r1 - r0, k), dtype=np.float32) * np.float32(1.0 / np.sqrt(k))
        out[r0:r1] = to_bf16_bits(w)
    return out
