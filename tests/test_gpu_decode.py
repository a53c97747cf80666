"""GPU parity of decode attention (a6 + a7) against the fp64 oracle: max |error|
<= 2e-3 and relative error <= 1e-2 where |reference| >= 0.2, on small shapes that
span several pages, stages and splits with ragged residual windows, plus the
degenerate cases (empty sequences, residual only, pages only)."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn
from bit_mixed_precision_channel_b200.cache import PagedKVCache

from _kv import assert_attention_close, oracle_unit, to_dev

pytestmark = pytest.mark.gpu


def _inputs(rng, L, cfg, outlier_scale=(8.0, 20.0), k_scale=1.0, v_scale=1.0):
    H, D = cfg.num_kv_heads, cfg.head_dim
    sig = np.exp(rng.standard_normal((H, D))).astype(np.float32)
    for h in range(H):
        sig[h, rng.choice(D, 5, replace=False)] *= rng.uniform(*outlier_scale, 5)
    K = syn.to_bits(rng.standard_normal((L, H, D)).astype(np.float32) * sig * k_scale, cfg.dtype)
    V = syn.to_bits(rng.standard_normal((L, H, D)).astype(np.float32) * v_scale, cfg.dtype)
    return K, V


def _run(cfg, lens, seed, max_pages=None, shuffle=False, q_scale=1.0, k_scale=1.0, v_scale=1.0, expect_err=0):
    """Prefill sequences of the given lengths, attend once; returns (out, oracle out)."""
    rng = np.random.default_rng(seed)
    P = cfg.page_tokens
    B = len(lens)
    max_pages = max_pages or max(1, max(L // P for L in lens))
    pool_pages = sum(L // P for L in lens) + 4
    page_order = np.random.default_rng(seed + 1).permutation(pool_pages) if shuffle else None
    cache = PagedKVCache(cfg, B, max_pages, pool_pages, page_order=page_order)
    inputs = []
    for b, L in enumerate(lens):
        K, V = _inputs(rng, L, cfg, k_scale=k_scale, v_scale=v_scale)
        inputs.append((K, V))
        if L:
            cache.prefill(b, to_dev(K, cfg.dtype), to_dev(V, cfg.dtype))
    q = syn.to_bits(rng.standard_normal((B, cfg.num_q_heads, cfg.head_dim)).astype(np.float32) * q_scale,
                    cfg.dtype)
    out = torch.full((B, cfg.num_q_heads, cfg.head_dim), float("nan"), device="cuda")
    q_dev = to_dev(q, cfg.dtype)
    cache.attend(q_dev, out)
    torch.cuda.synchronize()
    assert cache.err.item() == expect_err
    got = out.cpu().numpy()
    if expect_err:
        return got, None, cache
    want = np.zeros_like(got, dtype=np.float64)
    g = cfg.gqa
    for b, L in enumerate(lens):
        K, V = inputs[b]
        n = L // P
        for h in range(cfg.num_kv_heads):
            want[b, h * g:(h + 1) * g] = oracle_unit(cfg, K, V, n, K[n * P:L, h], V[n * P:L, h],
                                                     q[b, h * g:(h + 1) * g], h)
    cache.q_dev = q_dev
    return got, want, cache


SHAPES = [
    # gqa, dtype, P, k, lengths
    (4, kb.F16, 128, 32, [4096 + 77, 300, 128]),
    (4, kb.F16, 128, 16, [1000, 5 * 128, 1]),
    (8, kb.BF16, 128, 32, [2048 + 5, 130]),
    (8, kb.F16, 128, 32, [777, 256]),
    (1, kb.F16, 32, 16, [256, 250, 31]),
    (2, kb.BF16, 64, 64, [64 * 9 + 63, 100]),
    (4, kb.F16, 64, 0, [64 * 20 + 3]),
    (1, kb.BF16, 32, 128, [32 * 13 + 17]),
    (2, kb.F16, 128, 128, [128 * 3 + 127]),
    (4, kb.F16, 128, 64, [128 * 9 + 3, 77]),
]


@pytest.mark.parametrize("gqa,dtype,P,k,lens", SHAPES, ids=lambda v: str(v))
def test_decode_matches_oracle(gqa, dtype, P, k, lens):
    H = 2
    cfg = kb.Config(num_q_heads=gqa * H, num_kv_heads=H, page_tokens=P, num_boost=k, dtype=dtype)
    got, want, _ = _run(cfg, lens, seed=gqa * 100 + P + k + dtype)
    assert_attention_close(got, want, f"gqa{gqa} P{P} k{k}")


def test_split_count_does_not_change_result():
    """One sequence of 40 pages is cut across many CTAs (one or a few pages each) and
    merged by log-sum-exp; the weight counters are left at zero.  The same cache read
    through a 4000-entry page table and a fresh workspace gives the same answer."""
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=128, num_boost=32)
    got1, want, cache = _run(cfg, [128 * 40 + 9], seed=5)
    assert_attention_close(got1, want, "many splits")
    assert not cache.workspace[-4:].any()
    wide = torch.full((1, 4000), -1, dtype=torch.int32, device="cuda")
    wide[0, :40] = cache.page_table[0, :40]
    ws = torch.zeros(kb.decode_workspace_bytes(cfg, 1, 4000), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, 4, 128, device="cuda")
    kb.decode_attention(cfg, cache.pool, cache.q_dev, wide, cache.num_pages, cache.res_k, cache.res_v,
                        cache.res_len, out, ws)
    torch.cuda.synchronize()
    assert_attention_close(out.cpu().numpy(), want, "single split")


def test_empty_and_residual_only_sequences():
    cfg = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=128, num_boost=32)
    got, want, _ = _run(cfg, [0, 5, 128, 127, 129], seed=9)
    assert (got[0] == 0).all()
    assert_attention_close(got[1:], want[1:], "residual only / pages only")


def test_batch_above_one_pass_with_empty_runs():
    """More sequences than threads in a CTA (the weight line is summed in passes and the
    per-sequence lengths are cached from the located sequence on), with long runs of empty
    sequences that the item lists skip, some of them longer than the cache."""
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=32, num_boost=16)
    lens = [0] * 420
    for b, L in {0: 100, 1: 33, 150: 257, 151: 0, 290: 1, 291: 64, 419: 95}.items():
        lens[b] = L
    got, want, _ = _run(cfg, lens, seed=31)
    live = [b for b, L in enumerate(lens) if L]
    assert (np.delete(got, live, axis=0) == 0).all()
    assert_attention_close(got[live], want[live], "batch 420 with empty runs")


def test_shuffled_physical_pages():
    cfg = kb.Config(num_q_heads=4, num_kv_heads=2, page_tokens=128, num_boost=16)
    got, want, cache = _run(cfg, [128 * 20 + 50, 128 * 15], seed=13, shuffle=True)
    assert cache.host_pages[0] != sorted(cache.host_pages[0])
    assert_attention_close(got, want, "shuffled")


def test_peaked_attention_logits():
    """Large query norms make the softmax nearly one-hot: the hi/lo operand split has
    to carry the logits accurately enough for the tolerance."""
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=128, num_boost=32)
    got, want, _ = _run(cfg, [128 * 12 + 40], seed=21, q_scale=6.0)
    assert_attention_close(got, want, "peaked")


def test_bad_page_id_flags_error():
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=128, num_boost=32)
    cache = PagedKVCache(cfg, 1, max_pages=2, pool_pages=2)
    cache.page_table[0, 0] = 99
    cache.num_pages[0] = 1
    q = torch.zeros(1, 4, 128, dtype=torch.float16, device="cuda")
    out = torch.empty(1, 4, 128, device="cuda")
    cache.attend(q, out)
    torch.cuda.synchronize()
    assert cache.err.item() & kb.DEV_ERR_PAGE_RANGE


def test_bad_lengths_flag_error():
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=128, num_boost=32)
    cache = PagedKVCache(cfg, 2, max_pages=2, pool_pages=2)
    cache.num_pages[1] = 7  # more than max_pages
    q = torch.zeros(2, 4, 128, dtype=torch.float16, device="cuda")
    out = torch.zeros(2, 4, 128, device="cuda")
    cache.attend(q, out)
    torch.cuda.synchronize()
    assert cache.err.item() & kb.DEV_ERR_LENGTH


# ---------------------------------------------------------------- operand range

def test_large_queries_are_scaled_into_range():
    """fp16 cache, queries of magnitude ~10^4: q * key scale reaches ~10^5, past fp16's
    largest value.  The kernel carries q * 2^-e per head (|q * 2^-e| < 1), so the folded
    operands stay finite and the result matches the oracle (a nearly one-hot softmax)."""
    cfg = kb.Config(num_q_heads=4, num_kv_heads=2, page_tokens=128, num_boost=32)
    got, want, _ = _run(cfg, [128 * 6 + 40, 300], seed=41, q_scale=3000.0)
    assert_attention_close(got, want, "queries of magnitude 1e4")


@pytest.mark.parametrize("dtype", [kb.F16, kb.BF16])
def test_large_values_use_the_value_exponent(dtype):
    """Values of magnitude ~3000 (value scales ~2700): p * scale would pass 65504 in the
    fp16 PV operand without the per-warp value exponent.  Both sides are divided by the
    value magnitude before the comparison, so the tolerance applies to unit-sized values."""
    cfg = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=128, num_boost=16, dtype=dtype)
    got, want, _ = _run(cfg, [128 * 9 + 100, 77], seed=43, v_scale=1000.0)
    assert_attention_close(got / 1000.0, want / 1000.0, "values of magnitude 3e3")


def test_bf16_key_scales_beyond_fp16_flag_range():
    """bf16 keys of magnitude ~10^6: their scales and zero points cannot enter the fp16
    operands.  The call raises KVQ_DEV_ERR_RANGE instead of returning a silently wrong
    output."""
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=128, num_boost=32, dtype=kb.BF16)
    _run(cfg, [128 * 3 + 5], seed=45, k_scale=1e6, expect_err=kb.DEV_ERR_RANGE)
