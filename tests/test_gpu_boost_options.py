"""GPU parity of the boost options: the query-aware channel ranking (the MixKVQ
reading: channel range over the page times a query-relevance weight) and the per-head
boost count.  Every record byte must equal the
oracle's, through the prefill quantizer and through the residual flush; decode attention
over such records must match the oracle within the method's tolerance."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn

from _kv import assert_attention_close, ocfg, to_dev

pytestmark = pytest.mark.gpu


def _pages(rng, n_tok, H, dtype, ties=False):
    sig = np.exp(rng.standard_normal((H, 128))).astype(np.float32)
    for h in range(H):
        sig[h, rng.choice(128, 5, replace=False)] *= rng.uniform(8, 20, 5)
    K = rng.standard_normal((n_tok, H, 128)).astype(np.float32) * sig
    if ties:
        K = np.round(K)  # many channels share their range exactly
    V = rng.standard_normal((n_tok, H, 128)).astype(np.float32)
    return syn.to_bits(K, dtype), syn.to_bits(V, dtype)


def _options(rng, H, k, mode, ties=False):
    w = np.abs(rng.standard_normal((H, 128))).astype(np.float32) * 2
    if ties:
        w = np.round(w * 2) / 2
    kh = np.array([[k, k // 2, 0, 16 if k >= 16 else k][h % 4] for h in range(H)], np.int32)
    return (w if mode in ("query", "both") else None), (kh if mode in ("per_head", "both") else None)


def _dev(a, dtype):
    return None if a is None else torch.from_numpy(a).to("cuda")


@pytest.mark.parametrize("P,k,dtype,H,mode", [
    (128, 32, kb.F16, 4, "query"), (128, 32, kb.F16, 4, "per_head"), (128, 32, kb.BF16, 4, "both"),
    (64, 64, kb.F16, 2, "both"), (32, 16, kb.BF16, 3, "query"), (128, 128, kb.F16, 4, "per_head"),
    (128, 16, kb.F16, 4, "both"),
])
@pytest.mark.parametrize("ties", [False, True])
def test_boost_options_records_bit_exact(P, k, dtype, H, mode, ties):
    rng = np.random.default_rng(P + k + 7 * H + dtype + (100 if ties else 0) + len(mode))
    cfg = kb.Config(num_q_heads=H, num_kv_heads=H, page_tokens=P, num_boost=k, dtype=dtype)
    oc = ocfg(cfg)
    n_pages, pool_pages = 5, 9
    K, V = _pages(rng, n_pages * P, H, dtype, ties)
    w, kh = _options(rng, H, k, mode, ties)
    dst = [8, 1, 4, 0, 6]
    pool = torch.zeros(pool_pages * H * kb.page_bytes(cfg), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb.quantize_pages_ex(cfg, kb.Source.token_major(to_dev(K, dtype), cfg), kb.Source.token_major(to_dev(V, dtype), cfg),
                         torch.tensor(dst, dtype=torch.int32, device="cuda"), pool, err,
                         query_weight=_dev(w, dtype), boost_per_head=_dev(kh, dtype))
    torch.cuda.synchronize()
    assert err.item() == 0
    recs = pool.cpu().numpy().reshape(pool_pages, H, -1)
    payload = kb.page_layout(cfg)["payload_bytes"]
    for i, page in enumerate(dst):
        for h in range(H):
            want = oracle.quantize_page_ex(K[i * P:(i + 1) * P, h], V[i * P:(i + 1) * P, h], oc,
                                           n_boost=None if kh is None else int(kh[h]),
                                           weight=None if w is None else w[h])
            got = recs[page, h, :payload]
            assert np.array_equal(got, want[:payload]), \
                f"page {i} head {h}: {(got != want[:payload]).sum()} bytes differ"


@pytest.mark.parametrize("dtype", [kb.F16, kb.BF16])
def test_flush_with_boost_options_bit_exact(dtype):
    """Windows filled by appends and flushed with both options: the flushed records equal
    the oracle's records of the same P tokens."""
    from bit_mixed_precision_channel_b200.cache import PagedKVCache
    rng = np.random.default_rng(21 + dtype)
    B, H, P, k = 3, 4, 32, 16
    cfg = kb.Config(num_q_heads=8, num_kv_heads=H, page_tokens=P, num_boost=k, dtype=dtype)
    oc = ocfg(cfg)
    cache = PagedKVCache(cfg, B, max_pages=4, pool_pages=12)
    w, kh = _options(rng, H, k, "both")
    wd, khd = _dev(w, dtype), _dev(kh, dtype)
    streams = []
    for b, L in enumerate([5, 31, 20]):
        K, V = _pages(rng, L, H, dtype)
        cache.prefill(b, to_dev(K, dtype), to_dev(V, dtype))
        streams.append([K, V])
    for step in range(P):
        kn, vn = _pages(rng, B, H, dtype)  # one new token per sequence: [B][H][D]
        flushing = cache.reserve_flush_pages()
        cache.append(to_dev(kn, dtype), to_dev(vn, dtype))
        kb.flush_residual(cfg, cache.res_k, cache.res_v, cache.res_len, cache.new_page, cache.page_table,
                          cache.num_pages, cache.pool, cache.err, query_weight=wd, boost_per_head=khd)
        cache.commit_host(flushing)
        for b in range(B):
            streams[b][0] = np.concatenate([streams[b][0], kn[b:b + 1]])
            streams[b][1] = np.concatenate([streams[b][1], vn[b:b + 1]])
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    recs = cache.pool.cpu().numpy().reshape(12, H, -1)
    payload = kb.page_layout(cfg)["payload_bytes"]
    n = 0
    for b in range(B):
        K, V = streams[b]
        for i, page in enumerate(cache.host_pages[b]):
            for h in range(H):
                want = oracle.quantize_page_ex(K[i * P:(i + 1) * P, h], V[i * P:(i + 1) * P, h], oc,
                                               n_boost=int(kh[h]), weight=w[h])
                assert np.array_equal(recs[page, h, :payload], want[:payload]), (b, i, h)
                n += 1
    assert n == B * H  # every sequence flushed exactly one page


def test_decode_reads_records_with_per_head_counts():
    """Decode attention over records whose heads boost 32, 16, 0 and 16 of 32 rows (the
    unused rows are zero) matches the oracle's attention over the same records."""
    rng = np.random.default_rng(31)
    H, gqa, P, k = 4, 4, 128, 32
    cfg = kb.Config(num_q_heads=H * gqa, num_kv_heads=H, page_tokens=P, num_boost=k)
    oc = ocfg(cfg)
    L = P * 6
    K, V = _pages(rng, L, H, kb.F16)
    w, kh = _options(rng, H, k, "both")
    pool_pages = 6
    pool = torch.zeros(pool_pages * H * kb.page_bytes(cfg), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dst = torch.arange(6, dtype=torch.int32, device="cuda")
    kb.quantize_pages_ex(cfg, kb.Source.token_major(to_dev(K, kb.F16), cfg),
                         kb.Source.token_major(to_dev(V, kb.F16), cfg), dst, pool, err,
                         query_weight=_dev(w, kb.F16), boost_per_head=_dev(kh, kb.F16))
    q = syn.to_bits(rng.standard_normal((1, H * gqa, 128)).astype(np.float32), kb.F16)
    table = dst.view(1, 6)
    num = torch.tensor([6], dtype=torch.int32, device="cuda")
    res = torch.zeros(1, H, P, 128, dtype=torch.float16, device="cuda")
    rl = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(kb.decode_workspace_bytes(cfg, 1, 6), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, H * gqa, 128, device="cuda")
    kb.decode_attention(cfg, pool, to_dev(q, kb.F16), table, num, res, res, rl, out, ws, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    opool = np.zeros((pool_pages, H, oc.record_bytes), np.uint8)
    for i in range(6):
        for h in range(H):
            opool[i, h] = oracle.quantize_page_ex(K[i * P:(i + 1) * P, h], V[i * P:(i + 1) * P, h], oc,
                                                  n_boost=int(kh[h]), weight=w[h])
    got = out.cpu().numpy()[0]
    empty = np.zeros((0, 128), np.uint16)
    for h in range(H):
        want = oracle.decode_unit(opool, oc, h, list(range(6)), empty, empty, q[0, h * gqa:(h + 1) * gqa],
                                  1.0 / math.sqrt(128))
        assert_attention_close(got[h * gqa:(h + 1) * gqa], want, f"kv head {h} ({kh[h]} boosted)")


def test_per_head_count_out_of_range_flags_error():
    cfg = kb.Config(num_q_heads=2, num_kv_heads=2, page_tokens=32, num_boost=16)
    K, V = _pages(np.random.default_rng(1), 32, 2, kb.F16)
    pool = torch.zeros(2 * kb.page_bytes(cfg), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb.quantize_pages_ex(cfg, kb.Source.token_major(to_dev(K, kb.F16), cfg),
                         kb.Source.token_major(to_dev(V, kb.F16), cfg),
                         torch.zeros(1, dtype=torch.int32, device="cuda"), pool, err,
                         boost_per_head=torch.tensor([16, 17], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert err.item() & kb.DEV_ERR_LENGTH
