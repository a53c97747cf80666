"""Seeded synthetic inputs for the KV-cache workloads.

This module only draws random numbers and rounds them to the storage type; it holds
none of the quantization or attention arithmetic, so the CUDA path and the CPU
oracle can both take their inputs from it.

The pages measure on LongBench, InfiniteBench and seven reasoning tasks with trained
Qwen3 / LLaMA3 models; none of that is available here, so these generators stand in
for the KV tensors those runs would produce: keys with persistent outlier channels
(the reason Keys are quantized per channel, KIVI section 3) and Gaussian values and
queries, at the shapes of the five workloads below.

Every tensor comes from its own numpy PCG64 stream whose seed is derived from
(seed, tensor name, sequence, step), so any slice can be regenerated alone.
Tensors are returned as uint16 bit patterns of the storage type (fp16 or bf16).
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass

import numpy as np

F16 = 0
BF16 = 1


@dataclass(frozen=True)
class Workload:
    """One decode workload: cache shape, prompt lengths, key distribution, steps."""
    name: str
    batch: int
    Hq: int
    Hkv: int
    D: int
    P: int            # page tokens (= residual window capacity)
    G: int            # key group tokens
    k: int            # boosted key channels per page
    dtype: int        # F16 / BF16
    context: int      # prompt length (fixed lengths)
    steps: int        # decode steps
    key_dist: str     # "outliers" or "lognormal"
    ragged: tuple = ()  # (lo, hi) for uniform random prompt lengths
    shuffled_pages: bool = False
    n_outliers: int = 8
    outlier_scale: tuple = (10.0, 10.0)
    seed: int = 0

    @property
    def gqa(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    # batch 1, one head, 256 tokens, pages of 32 tokens, 8 outlier channels x10, 16 boosted
    "tiny": Workload("tiny", batch=1, Hq=1, Hkv=1, D=128, P=32, G=32, k=16, dtype=F16,
                     context=256, steps=1, key_dist="outliers", n_outliers=8,
                     outlier_scale=(10.0, 10.0)),
    # Llama-3-8B-shaped decode layer: 16 x 4096 tokens, 32 q / 8 kv heads, 25% boost
    "llama3_8b": Workload("llama3_8b", batch=16, Hq=32, Hkv=8, D=128, P=128, G=32, k=32,
                          dtype=F16, context=4096, steps=64, key_dist="lognormal",
                          n_outliers=5, outlier_scale=(8.0, 20.0)),
    # Qwen3-8B-shaped long context: 4 x 32768 tokens, 12.5% boost
    "qwen3_8b_long": Workload("qwen3_8b_long", batch=4, Hq=32, Hkv=8, D=128, P=128, G=32, k=16,
                              dtype=F16, context=32768, steps=32, key_dist="lognormal",
                              n_outliers=5, outlier_scale=(8.0, 20.0)),
    # Llama-3-70B-shaped large batch: 128 x 8192 tokens, 64 q / 8 kv heads, bf16, 25% boost
    "llama3_70b_batch": Workload("llama3_70b_batch", batch=128, Hq=64, Hkv=8, D=128, P=128,
                                 G=32, k=32, dtype=BF16, context=8192, steps=16,
                                 key_dist="lognormal", n_outliers=5, outlier_scale=(8.0, 20.0)),
    # Ragged serving: 64 sequences with lengths uniform in [1024, 32768], shuffled pages
    "ragged_serving": Workload("ragged_serving", batch=64, Hq=32, Hkv=8, D=128, P=128, G=32,
                               k=16, dtype=F16, context=0, steps=256, key_dist="lognormal",
                               ragged=(1024, 32768), shuffled_pages=True, n_outliers=5,
                               outlier_scale=(8.0, 20.0)),
}

ORDER = ["tiny", "llama3_8b", "qwen3_8b_long", "llama3_70b_batch", "ragged_serving"]


def _rng(w: Workload, tag: str, *ids: int) -> np.random.Generator:
    key = [w.seed, zlib.crc32(w.name.encode()), zlib.crc32(tag.encode())] + [int(i) for i in ids]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Rounds fp32 values to the storage type (nearest, ties to even) -> uint16 patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def from_bits(bits: np.ndarray, dtype: int) -> np.ndarray:
    """uint16 patterns -> fp32 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    if dtype == F16:
        return b.view(np.float16).astype(np.float32)
    return (b.astype(np.uint32) << 16).view(np.float32)


def lengths(w: Workload) -> np.ndarray:
    """Prompt length of every sequence."""
    if w.ragged:
        lo, hi = w.ragged
        return _rng(w, "lengths").integers(lo, hi + 1, size=w.batch).astype(np.int64)
    return np.full(w.batch, w.context, np.int64)


def key_channel_sigma(w: Workload) -> np.ndarray:
    """Per (kv head, channel) standard deviation of the keys, fixed for the layer.

    "outliers": 1 everywhere except n_outliers seeded channels per head at x scale.
    "lognormal": LogNormal(0, 1) per channel, then n_outliers seeded channels per head
    multiplied by U[lo, hi]."""
    r = _rng(w, "key_sigma")
    if w.key_dist == "outliers":
        sig = np.ones((w.Hkv, w.D), np.float32)
    else:
        sig = np.exp(r.standard_normal((w.Hkv, w.D))).astype(np.float32)
    lo, hi = w.outlier_scale
    for h in range(w.Hkv):
        ch = r.choice(w.D, size=w.n_outliers, replace=False)
        sig[h, ch] *= r.uniform(lo, hi, size=w.n_outliers).astype(np.float32)
    return sig


def keys(w: Workload, b: int, start: int, n: int, sigma: np.ndarray | None = None) -> np.ndarray:
    """Prompt keys of sequence b, tokens [start, start+n): [n][Hkv][D] patterns.

    Tokens are drawn in blocks of 256 so any aligned slice regenerates identically."""
    if sigma is None:
        sigma = key_channel_sigma(w)
    return to_bits(_blocks(w, "keys", b, start, n) * sigma[None], w.dtype)


def values(w: Workload, b: int, start: int, n: int) -> np.ndarray:
    """Prompt values of sequence b, tokens [start, start+n): [n][Hkv][D] patterns."""
    return to_bits(_blocks(w, "values", b, start, n), w.dtype)


_BLOCK = 256


def _blocks(w: Workload, tag: str, b: int, start: int, n: int) -> np.ndarray:
    out = np.empty((n, w.Hkv, w.D), np.float32)
    t = start
    while t < start + n:
        blk = t // _BLOCK
        x = _rng(w, tag, b, blk).standard_normal((_BLOCK, w.Hkv, w.D), dtype=np.float32)
        lo = t - blk * _BLOCK
        take = min(_BLOCK - lo, start + n - t)
        out[t - start:t - start + take] = x[lo:lo + take]
        t += take
    return out


def step_tokens(w: Workload, step: int, sigma: np.ndarray | None = None):
    """New key and value of every sequence at decode step `step`: [B][Hkv][D] each."""
    if sigma is None:
        sigma = key_channel_sigma(w)
    k = _rng(w, "step_keys", step).standard_normal((w.batch, w.Hkv, w.D), dtype=np.float32)
    v = _rng(w, "step_values", step).standard_normal((w.batch, w.Hkv, w.D), dtype=np.float32)
    return to_bits(k * sigma[None], w.dtype), to_bits(v, w.dtype)


def queries(w: Workload, step: int) -> np.ndarray:
    """Queries of decode step `step`: [B][Hq][D] patterns, N(0, 1)."""
    q = _rng(w, "queries", step).standard_normal((w.batch, w.Hq, w.D), dtype=np.float32)
    return to_bits(q, w.dtype)


def page_order(w: Workload, n_pages: int) -> np.ndarray:
    """Physical page ids handed out in order: identity, or a seeded permutation."""
    if w.shuffled_pages:
        return _rng(w, "page_order").permutation(n_pages).astype(np.int32)
    return np.arange(n_pages, dtype=np.int32)
