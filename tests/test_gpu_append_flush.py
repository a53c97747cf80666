"""kvq_append_flush (append and flush in one launch) against the two separate calls,
kvq_append_token then kvq_flush_residual, on identical caches: after every step the
windows, lengths, page tables, every pool byte, the error word and the arrival counters
must be identical.  The separate calls are themselves checked against the oracle
(test_gpu_quantize.py, and the workload tests run the fused call through
PagedKVCache.step against the oracle at full size)."""
import numpy as np
import pytest
import torch

from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn
from bit_mixed_precision_channel_b200.cache import PagedKVCache

pytestmark = pytest.mark.gpu


def _pair(cfg, B, max_pages, pool_pages, lens, seed):
    """Two caches with the same prompts (lengths `lens`)."""
    rng = np.random.default_rng(seed)
    dt = kb.torch_dtype(cfg.dtype)
    caches = [PagedKVCache(cfg, B, max_pages, pool_pages) for _ in range(2)]
    for b in range(B):
        L = int(lens[b])
        K = syn.to_bits((rng.standard_normal((L, cfg.num_kv_heads, cfg.head_dim)) * 3).astype(np.float32), cfg.dtype)
        V = syn.to_bits(rng.standard_normal((L, cfg.num_kv_heads, cfg.head_dim)).astype(np.float32), cfg.dtype)
        k = torch.from_numpy(K.view(np.int16)).view(dt).cuda()
        v = torch.from_numpy(V.view(np.int16)).view(dt).cuda()
        for c in caches:
            c.prefill(b, k, v)
    return caches


def _state(c: PagedKVCache):
    return [t.clone() for t in (c.res_k, c.res_v, c.res_len, c.num_pages, c.page_table, c.pool, c.err)]


def _same(a: PagedKVCache, b: PagedKVCache, what: str):
    names = ["res_k", "res_v", "res_len", "num_pages", "page_table", "pool", "err"]
    for n, x, y in zip(names, _state(a), _state(b)):
        if not torch.equal(x.view(torch.uint8) if x.dtype.is_floating_point else x,
                           y.view(torch.uint8) if y.dtype.is_floating_point else y):
            raise AssertionError(f"{what}: {n} differs")


def _step(fused: PagedKVCache, sep: PagedKVCache, kn, vn, new_page, **opts):
    for c in (fused, sep):
        c.new_page.copy_(new_page)
    kb.append_flush(fused.cfg, kn, vn, fused.res_k, fused.res_v, fused.res_len, fused.new_page,
                    fused.page_table, fused.num_pages, fused.pool, fused.counters, fused.err, **opts)
    kb.append_token(sep.cfg, kn, vn, sep.res_k, sep.res_v, sep.res_len, sep.err)
    kb.flush_residual(sep.cfg, sep.res_k, sep.res_v, sep.res_len, sep.new_page, sep.page_table,
                      sep.num_pages, sep.pool, sep.err, **opts)
    torch.cuda.synchronize()
    assert int(fused.counters.abs().sum()) == 0


@pytest.mark.parametrize("dtype,P,k", [(kb.F16, 32, 16), (kb.BF16, 64, 32), (kb.F16, 128, 32), (kb.F16, 32, 128)])
def test_fused_equals_separate_calls(dtype, P, k):
    cfg = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=P, num_boost=k, dtype=dtype)
    B = 6
    lens = [P - 1, P - 3, 2 * P, 3 * P - 2, 5, P + 7]
    max_pages, pool_pages = 8, 40
    fused, sep = _pair(cfg, B, max_pages, pool_pages, lens, seed=P + k)
    rng = np.random.default_rng(7)
    dt = kb.torch_dtype(dtype)
    next_page = 30
    for s in range(6):
        kn = torch.from_numpy(syn.to_bits((rng.standard_normal((B, 2, 128)) * 2).astype(np.float32), dtype)
                              .view(np.int16)).view(dt).cuda()
        vn = torch.from_numpy(syn.to_bits(rng.standard_normal((B, 2, 128)).astype(np.float32), dtype)
                              .view(np.int16)).view(dt).cuda()
        res = fused.res_len.cpu().tolist()
        ids = []
        for b in range(B):
            if res[b] + 1 == P:
                ids.append(next_page)
                next_page += 1
            else:
                ids.append(-1)
        _step(fused, sep, kn, vn, torch.tensor(ids, dtype=torch.int32))
        _same(fused, sep, f"step {s}")
    assert int(fused.err.item()) == 0
    assert next_page > 30  # some windows flushed


def test_fused_error_cases_match():
    """A window left full by a skipped flush (flushed now: RESIDUAL), a full window with
    no page (TABLE_FULL), a page id past the pool (PAGE_RANGE), a length past the window
    and a negative length (skipped, RESIDUAL / LENGTH), with per-head boost counts."""
    P = 32
    cfg = kb.Config(num_q_heads=4, num_kv_heads=2, page_tokens=P, num_boost=16, dtype=kb.F16)
    B = 7
    lens = [P - 1, P - 1, P - 1, 3, 3, 3, 2 * P]
    fused, sep = _pair(cfg, B, 6, 20, lens, seed=3)
    rng = np.random.default_rng(11)
    for c in (fused, sep):
        # b = 3: window already full, unflushed; b = 4: length past the window; b = 5: negative
        c.res_k[3].copy_(c.res_k[0])
        c.res_v[3].copy_(c.res_v[0])
        c.res_len[3] = P
        c.res_len[4] = P + 5
        c.res_len[5] = -2
    kn = torch.from_numpy(syn.to_bits(rng.standard_normal((B, 2, 128)).astype(np.float32), kb.F16)
                          .view(np.int16)).view(torch.float16).cuda()
    vn = kn.flip(0).contiguous()
    # b = 0 flushes into page 12, b = 1 has no page, b = 2 a page past the pool, b = 3 page 13
    new_page = torch.tensor([12, -1, 999, 13, -1, -1, -1], dtype=torch.int32)
    kh = torch.tensor([16, 9], dtype=torch.int32, device="cuda")
    _step(fused, sep, kn, vn, new_page, boost_per_head=kh)
    _same(fused, sep, "error step")
    err = int(fused.err.item())
    for bit in (kb.DEV_ERR_RESIDUAL, kb.DEV_ERR_TABLE_FULL, kb.DEV_ERR_PAGE_RANGE, kb.DEV_ERR_LENGTH):
        assert err & bit, (err, bit)
    assert fused.res_len.cpu().tolist()[:4] == [0, P, P, 0]
