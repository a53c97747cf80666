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
