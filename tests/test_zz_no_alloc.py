"""kvq_decode_attention_static: decode attention for callers that cannot allocate
device memory (their memory pool owns the GPU, or cudaMalloc is off limits on their
path), using the library's built-in static scratch instead of a workspace argument.

Checked through the C ABI against kvq_decode_attention on the same cache, on two calls
in a row (the second call reuses the scratch the first one left behind).  This file is
collected last so that a run stopping at the first failure has run everything else."""
import ctypes

import numpy as np
import pytest
import torch

from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn
from bit_mixed_precision_channel_b200.cache import PagedKVCache

from _kv import ATOL, RTOL, attention_errors, to_dev

pytestmark = pytest.mark.gpu


def _cache(cfg, lens, seed):
    rng = np.random.default_rng(seed)
    P = cfg.page_tokens
    cache = PagedKVCache(cfg, len(lens), max(L // P for L in lens) + 1, sum(L // P for L in lens) + 2)
    for b, L in enumerate(lens):
        sig = np.exp(rng.standard_normal((cfg.num_kv_heads, cfg.head_dim))).astype(np.float32)
        K = syn.to_bits(rng.standard_normal((L, cfg.num_kv_heads, cfg.head_dim)).astype(np.float32) * sig, cfg.dtype)
        V = syn.to_bits(rng.standard_normal((L, cfg.num_kv_heads, cfg.head_dim)).astype(np.float32), cfg.dtype)
        cache.prefill(b, to_dev(K, cfg.dtype), to_dev(V, cfg.dtype))
    return cache


@pytest.mark.parametrize("gqa,dtype", [(4, kb.F16), (8, kb.BF16)])
def test_static_scratch_matches_workspace_call_twice(gqa, dtype):
    cfg = kb.Config(num_q_heads=8 * gqa, num_kv_heads=8, page_tokens=128, num_boost=32, dtype=dtype)
    cache = _cache(cfg, [128 * 24 + 17, 128 * 7 + 100, 33], seed=gqa + dtype)
    B = 3
    rng = np.random.default_rng(99)
    for call in range(2):
        q = to_dev(syn.to_bits(rng.standard_normal((B, cfg.num_q_heads, 128)).astype(np.float32), dtype), dtype)
        want = torch.empty(B, cfg.num_q_heads, 128, device="cuda")
        got = torch.full_like(want, float("nan"))
        kb.decode_attention(cfg, cache.pool, q, cache.page_table, cache.num_pages, cache.res_k, cache.res_v,
                            cache.res_len, want, cache.workspace, err=cache.err)
        kb.decode_attention_static(cfg, cache.pool, q, cache.page_table, cache.num_pages, cache.res_k, cache.res_v,
                                   cache.res_len, got, err=cache.err)
        torch.cuda.synchronize()
        assert cache.err.item() == 0
        a, r = attention_errors(got.cpu().numpy(), want.cpu().numpy().astype(np.float64))
        assert a <= ATOL and r <= RTOL, f"call {call}: max abs {a:.2e}, max rel {r:.2e}"


def test_static_scratch_rejects_shapes_beyond_its_size():
    """Through the C ABI directly (the binding would refuse the placeholder tensors first):
    the shape check happens on the host, before anything is read."""
    cfg = kb.Config(num_q_heads=64, num_kv_heads=8, page_tokens=128, num_boost=32)
    batch, max_pages = 4096, 64
    assert kb.decode_workspace_bytes(cfg, batch, max_pages) > kb.STATIC_SCRATCH_BYTES
    t = torch.zeros(256, dtype=torch.int32, device="cuda")
    out = torch.zeros(256, dtype=torch.float32, device="cuda")
    pt = torch.zeros(batch, max_pages, dtype=torch.int32, device="cuda")
    p = t.data_ptr()
    status = kb.load().kvq_decode_attention_static(
        ctypes.byref(cfg.c()), p, 0, p, batch, pt.data_ptr(), max_pages, p, p, p, p, 0.088,
        out.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert status == 4  # KVQ_ERR_CAPACITY
