"""Host bookkeeping of PagedKVCache (CPU only): the free list, the flush-page
reservation that makes a decode step capturable, and the host mirrors of the window
lengths.  No kernel is launched; the buffers live on the CPU."""
import pytest
import torch

from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200.cache import PagedKVCache


def _cache(batch=3, pool_pages=6, order=None, P=32):
    cfg = kb.Config(num_q_heads=4, num_kv_heads=1, page_tokens=P, num_boost=16)
    return PagedKVCache(cfg, batch, max_pages=4, pool_pages=pool_pages, device="cpu", page_order=order)


def test_buffers_have_the_abi_shapes():
    c = _cache()
    assert c.page_table.shape == (3, 4) and (c.page_table == -1).all()
    assert c.pool.numel() == 6 * 1 * kb.page_bytes(c.cfg)
    assert c.res_k.shape == (3, 1, 32, 128) and c.res_k.dtype == torch.float16
    assert c.workspace.numel() >= kb.decode_workspace_bytes(c.cfg, 3, 4)


def test_free_list_follows_the_page_order_and_runs_out():
    c = _cache(order=[5, 4, 3, 2, 1, 0])
    assert c.take_pages(2) == [5, 4]
    assert c.take_pages(4) == [3, 2, 1, 0]
    with pytest.raises(RuntimeError):
        c.take_pages(1)


def test_page_order_must_be_a_permutation():
    with pytest.raises(ValueError):
        _cache(order=[0, 1, 2, 2, 4, 5])


def test_flush_pages_go_only_to_windows_that_fill_this_step():
    c = _cache(order=[5, 4, 3, 2, 1, 0])
    c.host_res_len = [31, 0, 31]          # after the append, sequences 0 and 2 hold P tokens
    flushing = c.reserve_flush_pages()
    assert flushing == [0, 2]
    assert c.new_page.tolist() == [5, -1, 4]
    c.commit_host(flushing)
    assert c.host_res_len == [0, 1, 0]
    assert c.host_pages == [[5], [], [4]]


def test_new_page_buffer_is_rewritten_only_when_it_changes():
    c = _cache()
    c.new_page.fill_(-7)                  # a stale device value would survive a skipped write
    assert c.reserve_flush_pages() == []  # nothing fills; the host mirror already says -1
    assert c.new_page.tolist() == [-7, -7, -7]
    c.host_res_len = [0, 31, 0]
    c.reserve_flush_pages()
    assert c.new_page.tolist() == [-1, 0, -1]


def test_a_window_never_exceeds_a_page():
    c = _cache()
    c.host_res_len = [31, 0, 0]
    with pytest.raises(AssertionError):
        c.commit_host([])                 # sequence 0 reached P tokens without a flush


def test_step_launches_the_flush_only_when_a_window_fills(monkeypatch):
    """PagedKVCache.step: append, then the flush only on a step where the host mirror says
    some window fills, then attention; the host lengths and pages advance either way."""
    c = _cache(order=[5, 4, 3, 2, 1, 0])
    calls = []
    monkeypatch.setattr(kb, "append_token", lambda *a, **k: calls.append("append"))
    monkeypatch.setattr(kb, "flush_residual", lambda *a, **k: calls.append("flush"))
    monkeypatch.setattr(kb, "decode_attention", lambda *a, **k: calls.append("attend"))
    q = torch.zeros(3, 4, 128, dtype=torch.float16)
    kn = torch.zeros(3, 1, 128, dtype=torch.float16)
    out = torch.zeros(3, 4, 128)
    c.host_res_len = [29, 0, 5]
    c.step(q, kn, kn, out)                 # 29 -> 30: nothing fills
    assert calls == ["append", "attend"] and c.host_res_len == [30, 1, 6]
    calls.clear()
    c.step(q, kn, kn, out)                 # 30 -> 31: still nothing
    c.step(q, kn, kn, out)                 # 31 -> 32 = P: sequence 0 flushes into page 5
    assert calls == ["append", "attend", "append", "flush", "attend"]
    assert c.host_res_len == [0, 3, 8] and c.host_pages == [[5], [], []]
    assert c.new_page.tolist() == [5, -1, -1]
