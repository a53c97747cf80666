"""kvq_decode_attention_static: decode attention for callers that cannot allocate
device memory (their memory pool owns the GPU, or cudaMalloc is off limits on their
path), using the library's built-in static scratch instead of a workspace argument.

Checked through the C ABI against the fp64 oracle and against kvq_decode_attention on
the same cache, on two calls in a row (the second reuses the scratch the first left
behind), across a change of shape whose arrival counters land where the previous call
left partial results, and with the device's free memory unchanged by a call.  This
file is collected last so that a run stopping at the first failure has run everything
else."""
import ctypes

import numpy as np
import pytest
import torch

from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn
from bit_mixed_precision_channel_b200.cache import PagedKVCache

from _kv import ATOL, RTOL, assert_attention_close, attention_errors, oracle_unit, to_dev

pytestmark = pytest.mark.gpu


def _cache(cfg, lens, seed):
    rng = np.random.default_rng(seed)
    P = cfg.page_tokens
    cache = PagedKVCache(cfg, len(lens), max(L // P for L in lens) + 1, sum(L // P for L in lens) + 2)
    raw = []
    for b, L in enumerate(lens):
        sig = np.exp(rng.standard_normal((cfg.num_kv_heads, cfg.head_dim))).astype(np.float32)
        K = syn.to_bits(rng.standard_normal((L, cfg.num_kv_heads, cfg.head_dim)).astype(np.float32) * sig, cfg.dtype)
        V = syn.to_bits(rng.standard_normal((L, cfg.num_kv_heads, cfg.head_dim)).astype(np.float32), cfg.dtype)
        cache.prefill(b, to_dev(K, cfg.dtype), to_dev(V, cfg.dtype))
        raw.append((K, V))
    return cache, raw


def _both(cfg, cache, q):
    B = q.shape[0]
    want = torch.empty(B, cfg.num_q_heads, 128, device="cuda")
    got = torch.full_like(want, float("nan"))
    kb.decode_attention(cfg, cache.pool, q, cache.page_table, cache.num_pages, cache.res_k, cache.res_v,
                        cache.res_len, want, cache.workspace, err=cache.err)
    kb.decode_attention_static(cfg, cache.pool, q, cache.page_table, cache.num_pages, cache.res_k, cache.res_v,
                               cache.res_len, got, err=cache.err)
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    return got.cpu().numpy(), want.cpu().numpy().astype(np.float64)


def test_batch_zero_call_resolves_the_scratch():
    """A call with batch 0 computes nothing and only looks the scratch up: the early
    set-up call a caller makes before its pool claims the device."""
    cfg = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=128, num_boost=32)
    status = kb.load().kvq_decode_attention_static(
        ctypes.byref(cfg.c()), None, 0, None, 0, None, 0, None, None, None, None, 0.088, None, None,
        torch.cuda.current_stream().cuda_stream)
    assert status == 0


@pytest.mark.parametrize("gqa,dtype", [(4, kb.F16), (8, kb.BF16)])
def test_static_scratch_matches_oracle_and_workspace_call_twice(gqa, dtype):
    cfg = kb.Config(num_q_heads=8 * gqa, num_kv_heads=8, page_tokens=128, num_boost=32, dtype=dtype)
    lens = [128 * 24 + 17, 128 * 7 + 100, 33]
    cache, raw = _cache(cfg, lens, seed=gqa + dtype)
    B, P = len(lens), cfg.page_tokens
    rng = np.random.default_rng(99)
    for call in range(2):
        qb = syn.to_bits(rng.standard_normal((B, cfg.num_q_heads, 128)).astype(np.float32), dtype)
        got, want = _both(cfg, cache, to_dev(qb, dtype))
        a, r = attention_errors(got, want)
        assert a <= ATOL and r <= RTOL, f"call {call} vs workspace call: max abs {a:.2e}, max rel {r:.2e}"
        for b, L in enumerate(lens):
            K, V = raw[b]
            n = L // P
            for h in (0, cfg.num_kv_heads - 1):
                ref = oracle_unit(cfg, K, V, n, K[n * P:L, h], V[n * P:L, h], qb[b, h * gqa:(h + 1) * gqa], h)
                assert_attention_close(got[b, h * gqa:(h + 1) * gqa], ref, f"call {call} seq {b} kv head {h}")


def test_shape_change_reuses_the_scratch_without_allocating():
    """A large call (64 sequences, GQA 8) fills the scratch with partial results; a small
    call (3 sequences) then puts its arrival counters where those partials were, and has
    to clear them.  Free device memory is the same before and after the second call."""
    big_cfg = kb.Config(num_q_heads=64, num_kv_heads=8, page_tokens=128, num_boost=32, dtype=kb.BF16)
    big, _ = _cache(big_cfg, [128 * 6 + 3 * i for i in range(64)], seed=3)
    qb = to_dev(syn.to_bits(np.random.default_rng(4).standard_normal((64, 64, 128)).astype(np.float32), kb.BF16),
                kb.BF16)
    got, want = _both(big_cfg, big, qb)
    a, r = attention_errors(got, want)
    assert a <= ATOL and r <= RTOL
    small_cfg = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=128, num_boost=16)
    assert kb.decode_workspace_bytes(small_cfg, 3, 20) < kb.decode_workspace_bytes(big_cfg, 64, 7)
    small, _ = _cache(small_cfg, [128 * 19 + 5, 128 * 3, 70], seed=5)
    qs = to_dev(syn.to_bits(np.random.default_rng(6).standard_normal((3, 8, 128)).astype(np.float32), kb.F16),
                kb.F16)
    want = torch.empty(3, 8, 128, device="cuda")
    got = torch.full_like(want, float("nan"))
    kb.decode_attention(small_cfg, small.pool, qs, small.page_table, small.num_pages, small.res_k, small.res_v,
                        small.res_len, want, small.workspace, err=small.err)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]  # every tensor of the call exists already
    kb.decode_attention_static(small_cfg, small.pool, qs, small.page_table, small.num_pages, small.res_k,
                               small.res_v, small.res_len, got, err=small.err)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert small.err.item() == 0
    got, want = got.cpu().numpy(), want.cpu().numpy().astype(np.float64)
    a, r = attention_errors(got, want)
    assert a <= ATOL and r <= RTOL, f"small call after a large one: max abs {a:.2e}, max rel {r:.2e}"
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"


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
        ctypes.byref(cfg.c()), p, 1, p, batch, pt.data_ptr(), max_pages, p, p, p, p, 0.088,
        out.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert status == 4  # KVQ_ERR_CAPACITY
