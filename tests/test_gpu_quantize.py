"""GPU parity of page quantization (a1-a3) and of the residual append/flush (a4-a5):
every byte of every checked record must equal the oracle's record."""
import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn

from _kv import kcfg, ocfg, to_dev

pytestmark = pytest.mark.gpu


def _random_pages(rng, n_pages, cfg, outliers=True, dtype=None):
    dtype = cfg.dtype if dtype is None else dtype
    P, H, D = cfg.page_tokens, cfg.num_kv_heads, cfg.head_dim
    sig = np.exp(rng.standard_normal((H, D))).astype(np.float32)
    if outliers:
        for h in range(H):
            sig[h, rng.choice(D, 5, replace=False)] *= rng.uniform(8, 20, 5)
    K = rng.standard_normal((n_pages * P, H, D)).astype(np.float32) * sig
    V = rng.standard_normal((n_pages * P, H, D)).astype(np.float32)
    return syn.to_bits(K, dtype), syn.to_bits(V, dtype)


def _pool(cfg, pool_pages):
    return torch.zeros(pool_pages * cfg.num_kv_heads * kb.page_bytes(cfg), dtype=torch.uint8, device="cuda")


def _records(pool, cfg, pool_pages):
    return pool.cpu().numpy().reshape(pool_pages, cfg.num_kv_heads, kb.page_bytes(cfg))


def _check_records(gpu_pool, cfg, K, V, dst, payload):
    oc = ocfg(cfg)
    P = cfg.page_tokens
    for i, page in enumerate(dst):
        for h in range(cfg.num_kv_heads):
            want = oracle.quantize_page(K[i * P:(i + 1) * P, h], V[i * P:(i + 1) * P, h], oc)
            got = gpu_pool[page, h]
            if not np.array_equal(got[:payload], want[:payload]):
                bad = np.nonzero(got[:payload] != want[:payload])[0]
                raise AssertionError(f"page {i} (phys {page}) head {h}: {bad.size} bytes differ, first at {bad[0]}")


CASES = [
    # (P, k, dtype, gqa-irrelevant Hkv)
    (128, 32, kb.F16, 2), (128, 16, kb.F16, 2), (128, 0, kb.F16, 1), (128, 128, kb.F16, 1),
    (64, 32, kb.F16, 2), (32, 16, kb.F16, 3), (128, 32, kb.BF16, 2), (32, 16, kb.BF16, 1),
    (64, 64, kb.BF16, 2),
]


@pytest.mark.parametrize("P,k,dtype,H", CASES, ids=lambda v: str(v))
def test_quantize_pages_bit_exact(P, k, dtype, H):
    rng = np.random.default_rng(P * 1000 + k * 10 + dtype)
    cfg = kb.Config(num_q_heads=H, num_kv_heads=H, page_tokens=P, num_boost=k, dtype=dtype)
    n_pages, pool_pages = 7, 12
    K, V = _random_pages(rng, n_pages, cfg)
    dst = [9, 0, 3, 11, 5, 1, 7]  # scattered physical pages
    pool = _pool(cfg, pool_pages)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb.quantize_pages(cfg, kb.Source.token_major(to_dev(K, dtype), cfg), kb.Source.token_major(to_dev(V, dtype), cfg),
                      torch.tensor(dst, dtype=torch.int32, device="cuda"), pool, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    recs = _records(pool, cfg, pool_pages)
    _check_records(recs, cfg, K, V, dst, kb.page_layout(cfg)["payload_bytes"])
    # pages not named in dst stay untouched
    for page in set(range(pool_pages)) - set(dst):
        assert not recs[page].any()


@pytest.mark.parametrize("dtype", [kb.F16, kb.BF16])
def test_separate_calls_equal_fused_call(dtype):
    rng = np.random.default_rng(77 + dtype)
    cfg = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=128, num_boost=32, dtype=dtype)
    K, V = _random_pages(rng, 5, cfg)
    dst = torch.tensor([4, 2, 0, 1, 3], dtype=torch.int32, device="cuda")
    ks = kb.Source.token_major(to_dev(K, dtype), cfg)
    vs = kb.Source.token_major(to_dev(V, dtype), cfg)
    a, b = _pool(cfg, 5), _pool(cfg, 5)
    kb.quantize_pages(cfg, ks, vs, dst, a)
    kb.select_boost_channels(cfg, ks, dst, b)
    kb.quantize_page_keys(cfg, ks, dst, b)
    kb.quantize_values(cfg, vs, dst, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_constant_and_degenerate_pages():
    """Constant channels (scale 0), all-equal magnitudes (every channel ties), zeros."""
    cfg = kb.Config(num_q_heads=1, num_kv_heads=1, page_tokens=32, num_boost=16, dtype=kb.F16)
    P, D = 32, 128
    pages_k = [np.zeros((P, 1, D), np.float32), np.full((P, 1, D), 1.5, np.float32),
               np.tile(np.where(np.arange(D) % 2, -2.0, 2.0).astype(np.float32), (P, 1, 1))]
    pages_v = [np.zeros((P, 1, D), np.float32), np.full((P, 1, D), -0.75, np.float32),
               np.tile(np.linspace(-1, 1, D, dtype=np.float32), (P, 1, 1))]
    K = syn.to_bits(np.concatenate(pages_k), kb.F16)
    V = syn.to_bits(np.concatenate(pages_v), kb.F16)
    pool = _pool(cfg, 3)
    kb.quantize_pages(cfg, kb.Source.token_major(to_dev(K, kb.F16), cfg), kb.Source.token_major(to_dev(V, kb.F16), cfg),
                      torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda"), pool)
    torch.cuda.synchronize()
    _check_records(_records(pool, cfg, 3), cfg, K, V, [0, 1, 2], kb.page_layout(cfg)["payload_bytes"])


def test_rounding_ties_take_the_exact_path():
    """Codes that land exactly on k + 1/2 (unit scales: groups spanning 0..3 and 0..15)
    must round half to even like the IEEE divide followed by rint, for keys (2- and 4-bit)
    and values; the kernel's multiply-by-reciprocal path hands such elements to the
    divide."""
    cfg = kb.Config(num_q_heads=1, num_kv_heads=1, page_tokens=32, num_boost=16, dtype=kb.F16)
    P, D = 32, 128
    t = np.arange(P)[:, None]
    c = np.arange(D)[None, :]
    hi = np.concatenate([[0.0, 15.0], np.arange(15) + 0.5, np.arange(15) + 0.25])  # 32 values, 0..15
    lo = np.array([0.0, 3.0, 0.5, 1.5, 2.5, 1.0, 2.0, 0.25])                       # 8 values, 0..3
    K = np.where(c < 16, hi[(t + c) % 32], lo[(t + c) % 8]).astype(np.float32)[:, None, :]
    V = lo[(t + 3 * c) % 8].astype(np.float32)[:, None, :]
    K, V = syn.to_bits(K, kb.F16), syn.to_bits(V, kb.F16)
    pool = _pool(cfg, 1)
    kb.quantize_pages(cfg, kb.Source.token_major(to_dev(K, kb.F16), cfg), kb.Source.token_major(to_dev(V, kb.F16), cfg),
                      torch.tensor([0], dtype=torch.int32, device="cuda"), pool)
    torch.cuda.synchronize()
    _check_records(_records(pool, cfg, 1), cfg, K, V, [0], kb.page_layout(cfg)["payload_bytes"])
    # the ties are really there: a unit-scale group rounds 0.5 / 1.5 / 2.5 to 0 / 2 / 2
    codes, _, _ = oracle.quant_group(V[:8, 0, 0], 2, kb.F16)
    assert list(codes) == [0, 3, 0, 2, 2, 1, 2, 0]


def test_bad_destination_page_sets_error_and_writes_nothing():
    cfg = kb.Config(num_q_heads=1, num_kv_heads=1, page_tokens=32, num_boost=16)
    rng = np.random.default_rng(3)
    K, V = _random_pages(rng, 2, cfg)
    pool = _pool(cfg, 2)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb.quantize_pages(cfg, kb.Source.token_major(to_dev(K, cfg.dtype), cfg),
                      kb.Source.token_major(to_dev(V, cfg.dtype), cfg),
                      torch.tensor([5, -1], dtype=torch.int32, device="cuda"), pool, err)
    torch.cuda.synchronize()
    assert err.item() & kb.DEV_ERR_PAGE_RANGE
    assert not pool.any()


def test_zero_pages_is_a_no_op():
    cfg = kb.Config(num_q_heads=1, num_kv_heads=1, page_tokens=32, num_boost=16)
    pool = _pool(cfg, 1)
    x = torch.zeros(32, 1, 128, dtype=torch.float16, device="cuda")
    kb.quantize_pages(cfg, kb.Source.token_major(x, cfg), kb.Source.token_major(x, cfg),
                      torch.zeros(0, dtype=torch.int32, device="cuda"), pool)
    torch.cuda.synchronize()
    assert not pool.any()


@pytest.mark.parametrize("dtype", [kb.F16, kb.BF16])
def test_append_and_flush_match_oracle(dtype):
    """Append tokens until windows fill, flush them into reserved pages; the residual
    window, page table and the flushed records must equal the oracle's."""
    from bit_mixed_precision_channel_b200.cache import PagedKVCache
    rng = np.random.default_rng(11 + dtype)
    B, H, P = 3, 2, 32
    cfg = kb.Config(num_q_heads=4, num_kv_heads=H, page_tokens=P, num_boost=16, dtype=dtype)
    oc = ocfg(cfg)
    cache = PagedKVCache(cfg, B, max_pages=8, pool_pages=16)
    ocache = oracle.OracleCache(oc, B, 16)
    lens = [40, 95, 64]
    for b, L in enumerate(lens):
        K, V = _random_pages(rng, (L + P - 1) // P, cfg)
        K, V = K[:L], V[:L]
        cache.prefill(b, to_dev(K, dtype), to_dev(V, dtype))
        ocache.prefill(b, K, V, cache.host_pages[b])
    for step in range(2 * P):
        kn = syn.to_bits(rng.standard_normal((B, H, 128)).astype(np.float32) * 3, dtype)
        vn = syn.to_bits(rng.standard_normal((B, H, 128)).astype(np.float32), dtype)
        flushing = cache.reserve_flush_pages()
        cache.append(to_dev(kn, dtype), to_dev(vn, dtype))
        cache.flush()
        new = cache.new_page.cpu().numpy()
        cache.commit_host(flushing)
        ocache.append(kn, vn)
        assert sorted(ocache.flush(new)) == sorted(flushing)
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    for b in range(B):
        assert cache.host_pages[b] == ocache.seqs[b].pages
        assert cache.num_pages[b].item() == len(ocache.seqs[b].pages)
        assert cache.page_table[b, :len(ocache.seqs[b].pages)].tolist() == ocache.seqs[b].pages
        r = ocache.res_len(b)
        assert cache.res_len[b].item() == r
        for h in range(H):
            got = cache.res_k[b, h, :r].view(torch.int16).cpu().numpy().view(np.uint16)
            want = np.stack(ocache.seqs[b].res_k[h]) if r else np.zeros((0, 128), np.uint16)
            assert np.array_equal(got, want)
    recs = cache.pool.cpu().numpy().reshape(16, H, -1)
    payload = kb.page_layout(cfg)["payload_bytes"]
    for b in range(B):
        for page in ocache.seqs[b].pages:
            for h in range(H):
                assert np.array_equal(recs[page, h, :payload], ocache.pool[page, h, :payload]), (b, page, h)


def test_append_into_full_window_flags_error():
    from bit_mixed_precision_channel_b200.cache import PagedKVCache
    cfg = kb.Config(num_q_heads=1, num_kv_heads=1, page_tokens=32, num_boost=16)
    cache = PagedKVCache(cfg, 1, max_pages=2, pool_pages=2)
    cache.res_len.fill_(32)
    x = torch.zeros(1, 1, 128, dtype=torch.float16, device="cuda")
    cache.append(x, x)
    torch.cuda.synchronize()
    assert cache.err.item() & kb.DEV_ERR_RESIDUAL
    assert cache.res_len.item() == 32


def test_flush_with_full_table_flags_error():
    from bit_mixed_precision_channel_b200.cache import PagedKVCache
    cfg = kb.Config(num_q_heads=1, num_kv_heads=1, page_tokens=32, num_boost=16)
    cache = PagedKVCache(cfg, 1, max_pages=1, pool_pages=3)
    cache.num_pages.fill_(1)
    cache.res_len.fill_(32)
    cache.new_page.fill_(2)
    cache.flush()
    torch.cuda.synchronize()
    assert cache.err.item() & kb.DEV_ERR_TABLE_FULL
    assert cache.res_len.item() == 32 and cache.num_pages.item() == 1
    assert not cache.pool.any()
