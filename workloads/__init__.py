"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and bench.py.

This module only draws random numbers and shapes them into the workloads the
TurboQuant pages describe (KV caches of a Llama-3.1-8B-shaped layer, serving and
long-context decode sweeps, a vector-search database).  It contains none of the
quantizer's arithmetic: no rotation, codebook, estimator or attention code lives
here, so both the CPU oracle and the CUDA path can take their inputs from it
without sharing any of the method's code.

Every draw comes from ``numpy.random.Generator(PCG64(SeedSequence([seed, stream])))``;
``stream`` separates independent draws (keys, values, queries, outlier channels, ...)
made from the same data seed.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# stream indices: one independent generator per kind of draw
STREAM_KEYS = 1
STREAM_VALUES = 2
STREAM_QUERIES = 3
STREAM_KEY_OUTLIERS = 4
STREAM_VALUE_OUTLIERS = 5
STREAM_KEY_SCALE = 6
STREAM_VALUE_SCALE = 7
STREAM_NEW_KEYS = 8
STREAM_NEW_VALUES = 9
STREAM_DB = 10


def generator(seed: int, stream: int) -> np.random.Generator:
    """Independent PCG64 generator for (data seed, stream index)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


def gaussian(shape, seed: int, stream: int) -> np.ndarray:
    """i.i.d. N(0, 1) float64 array."""
    return generator(seed, stream).standard_normal(size=shape)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to the nearest bfloat16 (ties to even) and return
    them as float32 (every bfloat16 is exactly representable in float32)."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the 16 dropped bits; NaN/Inf do not occur in these workloads
    rounding = ((u >> 16) & 1) + 0x7FFF
    r = ((u + rounding) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(f.shape)


def outlier_channels(n_heads: int, dim: int, count: int, seed: int, stream: int) -> np.ndarray:
    """Per head, ``count`` distinct channel indices chosen once from the seed stream."""
    g = generator(seed, stream)
    return np.stack([np.sort(g.choice(dim, size=count, replace=False)) for _ in range(n_heads)])


def apply_outliers(x: np.ndarray, channels: np.ndarray, factor: float) -> np.ndarray:
    """Scale the chosen channels of each head by ``factor``.  ``x`` is [..., H, T, D]."""
    y = x.copy()
    for h in range(channels.shape[0]):
        y[..., h, :, channels[h]] *= factor
    return y


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Shapes of one decode-attention workload (per layer)."""
    name: str
    batch: int
    kv_heads: int
    q_heads: int
    head_dim: int
    context: int
    # channel groups [(offset, width, key_bits, value_bits)]
    groups: tuple
    outliers: int = 0          # outlier channels per head
    outlier_factor: float = 8.0
    lognormal_sigma: float = 0.0  # per-(batch, token) norm scale ~ logN(0, sigma)
    new_tokens: int = 1        # tokens appended per sequence before the decode step
    decode_steps: int = 1

    @property
    def token_heads(self) -> int:
        return self.batch * self.kv_heads * self.context


# The workloads named by the TurboQuant pages' experiments, shaped as synthetic stand-ins.
TOY = dict(name="toy", d=128, bits=3, n_keys=4096, n_queries=16)

LLAMA_DECODE = DecodeWorkload(
    name="llama3.1-8b-layer-decode-32k", batch=1, kv_heads=8, q_heads=32, head_dim=128,
    context=32768, groups=((0, 128, 4, 4),), outliers=4)

SERVING_3P5 = DecodeWorkload(
    name="serving-decode-3.5bit", batch=64, kv_heads=8, q_heads=32, head_dim=128,
    context=8192, groups=((0, 64, 4, 4), (64, 64, 3, 3)), lognormal_sigma=0.5)

LONG_2P5 = DecodeWorkload(
    name="long-context-2.5bit-128k", batch=1, kv_heads=8, q_heads=32, head_dim=128,
    context=131072, groups=((0, 64, 3, 3), (64, 64, 2, 2)), outliers=4, decode_steps=32)

SEARCH_1536 = dict(name="search-d1536", d=1536, bits=4, n_db=1_000_000, n_queries=1000, k=10)
SEARCH_200 = dict(name="search-d200", d=200, bits=4, n_db=1_000_000, n_queries=1000, k=10)
SEARCH_3072 = dict(name="search-d3072", d=3072, bits=4, n_db=1_000_000, n_queries=1000, k=10)


def toy_inputs(seed: int = 0, n_keys: int = 4096, n_queries: int = 16, d: int = 128):
    """Keys N(0,1) float32 [n_keys, d] and queries N(0,1) float32 [n_queries, d]."""
    keys = gaussian((n_keys, d), seed, STREAM_KEYS).astype(np.float32)
    queries = gaussian((n_queries, d), seed, STREAM_QUERIES).astype(np.float32)
    return keys, queries


def decode_kv(w: DecodeWorkload, seed: int = 0, context: Optional[int] = None,
              batch: Optional[int] = None):
    """bf16-valued K and V caches [B, Hkv, T, D] (returned as float32 arrays holding
    bf16 values), following the workload's value distribution."""
    T = w.context if context is None else context
    B = w.batch if batch is None else batch
    shape = (B, w.kv_heads, T, w.head_dim)
    k = gaussian(shape, seed, STREAM_KEYS)
    v = gaussian(shape, seed, STREAM_VALUES)
    if w.outliers:
        k = apply_outliers(k, outlier_channels(w.kv_heads, w.head_dim, w.outliers, seed,
                                               STREAM_KEY_OUTLIERS), w.outlier_factor)
        v = apply_outliers(v, outlier_channels(w.kv_heads, w.head_dim, w.outliers, seed,
                                               STREAM_VALUE_OUTLIERS), w.outlier_factor)
    if w.lognormal_sigma:
        sk = generator(seed, STREAM_KEY_SCALE).lognormal(0.0, w.lognormal_sigma, size=(B, 1, T, 1))
        sv = generator(seed, STREAM_VALUE_SCALE).lognormal(0.0, w.lognormal_sigma, size=(B, 1, T, 1))
        k = k * sk
        v = v * sv
    return round_bf16(k), round_bf16(v)


def decode_queries(w: DecodeWorkload, seed: int = 0, batch: Optional[int] = None, step: int = 0):
    """bf16-valued queries [B, Hq, D] for decode step ``step``."""
    B = w.batch if batch is None else batch
    q = gaussian((B, w.q_heads, w.head_dim), seed + 7919 * step, STREAM_QUERIES)
    return round_bf16(q)


def decode_new_tokens(w: DecodeWorkload, seed: int = 0, batch: Optional[int] = None, step: int = 0):
    """bf16-valued new K/V rows [B, Hkv, new_tokens, D] appended before a decode step."""
    B = w.batch if batch is None else batch
    shape = (B, w.kv_heads, w.new_tokens, w.head_dim)
    k = gaussian(shape, seed + 7919 * step, STREAM_NEW_KEYS)
    v = gaussian(shape, seed + 7919 * step, STREAM_NEW_VALUES)
    if w.lognormal_sigma:
        k = k * generator(seed + 7919 * step, STREAM_KEY_SCALE).lognormal(0.0, w.lognormal_sigma, size=(B, 1, w.new_tokens, 1))
        v = v * generator(seed + 7919 * step, STREAM_VALUE_SCALE).lognormal(0.0, w.lognormal_sigma, size=(B, 1, w.new_tokens, 1))
    return round_bf16(k), round_bf16(v)


def unit_gaussian(n: int, d: int, seed: int, stream: int, start: int = 0) -> np.ndarray:
    """Rows ``start .. start+n`` of an i.i.d. Gaussian matrix, each row normalised to unit
    norm (float32).  Rows are drawn in chunks of 65536 from per-chunk generators so any
    row range can be regenerated without drawing the rows before it."""
    chunk = 65536
    out = np.empty((n, d), dtype=np.float32)
    r = start
    while r < start + n:
        c = r // chunk
        lo = c * chunk
        hi = min(lo + chunk, start + n)
        g = generator(seed, stream * 1_000_003 + c)
        block = g.standard_normal(size=(hi - lo, d))
        a = r - lo
        rows = block[a:]
        rows = rows / np.linalg.norm(rows, axis=1, keepdims=True)
        out[r - start: r - start + rows.shape[0]] = rows.astype(np.float32)
        r = hi
    return out


def search_inputs(d: int, n_db: int, n_queries: int, seed: int = 0):
    """Unit-norm Gaussian database [n_db, d] and queries [n_queries, d] (float32)."""
    return (unit_gaussian(n_db, d, seed, STREAM_DB),
            unit_gaussian(n_queries, d, seed, STREAM_QUERIES))
