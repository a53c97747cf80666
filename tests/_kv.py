"""Helpers shared by the parity tests: conversions between the seeded uint16 inputs,
torch device tensors and the oracle, and the attention tolerance of the method
(max |error| <= 2e-3; relative error <= 1e-2 wherever |reference| >= 0.2)."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn

ATOL = 2e-3
RTOL = 1e-2
REL_FLOOR = ATOL / RTOL  # 0.2: below it the absolute bound is the stricter one


def kcfg(w: syn.Workload, **over) -> kb.Config:
    d = dict(head_dim=w.D, num_q_heads=w.Hq, num_kv_heads=w.Hkv, page_tokens=w.P, key_group=w.G,
             num_boost=w.k, dtype=w.dtype)
    d.update(over)
    return kb.Config(**d)


def ocfg(c: kb.Config) -> oracle.Cfg:
    return oracle.Cfg(D=c.head_dim, Hq=c.num_q_heads, Hkv=c.num_kv_heads, P=c.page_tokens, G=c.key_group,
                      k=c.num_boost, dtype=c.dtype)


def to_dev(bits: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(kb.torch_dtype(dtype))
    return t.to(device)


def attention_errors(got: np.ndarray, want: np.ndarray):
    err = np.abs(got.astype(np.float64) - want)
    mask = np.abs(want) >= REL_FLOOR
    rel = float((err[mask] / np.abs(want[mask])).max()) if mask.any() else 0.0
    return float(err.max()), rel


def assert_attention_close(got: np.ndarray, want: np.ndarray, what: str = ""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    a, r = attention_errors(got, want)
    assert a <= ATOL and r <= RTOL, f"{what}: max abs {a:.3e} (<= {ATOL}), max rel {r:.3e} (<= {RTOL})"


def oracle_unit(cfg: kb.Config, K: np.ndarray, V: np.ndarray, n_pages: int, res_k: np.ndarray,
                res_v: np.ndarray, q_heads: np.ndarray, kvh: int, sm_scale: float | None = None) -> np.ndarray:
    """Oracle attention of one (sequence, kv head) from raw inputs: quantizes the
    sequence's first n_pages pages of head kvh itself, then runs decode_unit.
    K, V: [L][Hkv][D] patterns (L >= n_pages*P); res_k/res_v: [r][D] patterns;
    q_heads: [gqa][D] patterns."""
    oc = ocfg(cfg)
    P = cfg.page_tokens
    pool = np.zeros((max(n_pages, 1), cfg.num_kv_heads, oc.record_bytes), np.uint8)
    for i in range(n_pages):
        pool[i, kvh] = oracle.quantize_page(K[i * P:(i + 1) * P, kvh], V[i * P:(i + 1) * P, kvh], oc)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    return oracle.decode_unit(pool, oc, kvh, list(range(n_pages)), res_k, res_v, q_heads, sm_scale)
