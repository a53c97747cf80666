"""Device buffers and host bookkeeping of one layer's paged 2-bit KV cache.

PagedKVCache owns the caller-side state the C ABI expects (page pool, page table,
page counts, residual windows, decode workspace, device error word) plus a host free
list of physical pages.  Its methods only allocate, track page ids and call the
library; every transformation of the data happens in the library's kernels.

The decode step follows the pipeline of the KIVI article (section 3: recent tokens
kept in full precision, streaming append) with Kitty's paged layout: append the new
token to the residual window, flush the window into a fresh page when it holds a
whole page, then attend over pages + window.
"""
from __future__ import annotations

import torch

from . import binding as kb


class PagedKVCache:
    def __init__(self, cfg: kb.Config, batch: int, max_pages: int, pool_pages: int,
                 device: str | torch.device = "cuda", page_order=None):
        self.cfg = cfg
        self.batch = batch
        self.max_pages = max_pages
        self.pool_pages = pool_pages
        self.device = torch.device(device)
        H, P, D = cfg.num_kv_heads, cfg.page_tokens, cfg.head_dim
        dt = kb.torch_dtype(cfg.dtype)
        self.record_bytes = kb.page_bytes(cfg)
        self.pool = torch.zeros(pool_pages * H * self.record_bytes, dtype=torch.uint8, device=self.device)
        self.page_table = torch.full((batch, max_pages), -1, dtype=torch.int32, device=self.device)
        self.num_pages = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.res_len = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.res_k = torch.zeros(batch, H, P, D, dtype=dt, device=self.device)
        self.res_v = torch.zeros(batch, H, P, D, dtype=dt, device=self.device)
        ws = kb.decode_workspace_bytes(cfg, batch, max_pages)
        self.workspace = torch.zeros(max(ws, 256), dtype=torch.uint8, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.new_page = torch.full((batch,), -1, dtype=torch.int32, device=self.device)
        self.counters = torch.zeros(batch, dtype=torch.int32, device=self.device)  # append_flush arrivals
        # host mirrors used to hand out pages
        order = list(range(pool_pages)) if page_order is None else [int(x) for x in page_order]
        if sorted(order) != list(range(pool_pages)):
            raise ValueError("page_order must be a permutation of range(pool_pages)")
        self.free = order[::-1]  # pop() hands out order[0] first
        self.host_pages = [[] for _ in range(batch)]
        self.host_res_len = [0] * batch
        self.host_new_page = [-1] * batch  # what the device new_page buffer holds

    # ---------------------------------------------------------------- allocation
    def take_pages(self, n: int) -> list:
        if n > len(self.free):
            raise RuntimeError("page pool exhausted")
        return [self.free.pop() for _ in range(n)]

    # ---------------------------------------------------------------- prefill
    def prefill(self, b: int, k: torch.Tensor, v: torch.Tensor, stream=None):
        """k, v: [L][Hkv][D] on the device.  floor(L/P) pages are quantized, the
        remaining L mod P tokens are copied into the residual window."""
        P = self.cfg.page_tokens
        L = k.shape[0]
        n_full = L // P
        if len(self.host_pages[b]) + n_full > self.max_pages:
            raise RuntimeError("page table full")
        pages = self.take_pages(n_full)
        if n_full:
            dst = torch.tensor(pages, dtype=torch.int32, device=self.device)
            kb.quantize_pages(self.cfg, kb.Source.token_major(k, self.cfg), kb.Source.token_major(v, self.cfg),
                              dst, self.pool, self.err, stream)
            start = len(self.host_pages[b])
            self.page_table[b, start:start + n_full] = dst
        self.host_pages[b] += pages
        self.num_pages[b] = len(self.host_pages[b])
        r = L - n_full * P
        if r:
            self.res_k[b, :, :r] = k[n_full * P:].transpose(0, 1)
            self.res_v[b, :, :r] = v[n_full * P:].transpose(0, 1)
        self.res_len[b] = r
        self.host_res_len[b] = r

    def prefill_batch(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        """All sequences at once with the same prompt length L (a multiple of P):
        k, v: [B][L][Hkv][D] contiguous.  One quantize launch for every page."""
        B, L = k.shape[0], k.shape[1]
        P = self.cfg.page_tokens
        assert B == self.batch and L % P == 0 and k.is_contiguous() and v.is_contiguous()
        n = L // P
        pages = self.take_pages(B * n)
        dst = torch.tensor(pages, dtype=torch.int32, device=self.device)
        flat_k, flat_v = k.view(B * L, *k.shape[2:]), v.view(B * L, *v.shape[2:])
        kb.quantize_pages(self.cfg, kb.Source.token_major(flat_k, self.cfg), kb.Source.token_major(flat_v, self.cfg),
                          dst, self.pool, self.err, stream)
        self.page_table[:, :n] = dst.view(B, n)
        self.num_pages.fill_(n)
        self.res_len.zero_()
        for b in range(B):
            self.host_pages[b] += pages[b * n:(b + 1) * n]
            self.host_res_len[b] = 0
        return dst

    # ---------------------------------------------------------------- decode step
    def reserve_flush_pages(self) -> list:
        """Before a step: a fresh page for every sequence whose window will be full
        after this step's append; returns the sequences that will flush.  The device
        buffer is only written when its contents change."""
        P = self.cfg.page_tokens
        flushing = [b for b in range(self.batch) if self.host_res_len[b] + 1 == P]
        ids = [-1] * self.batch
        for b in flushing:
            ids[b] = self.take_pages(1)[0]
        if ids != self.host_new_page:
            self.new_page.copy_(torch.tensor(ids, dtype=torch.int32), non_blocking=False)
            self.host_new_page = ids
        return flushing

    def commit_host(self, flushing: list):
        P = self.cfg.page_tokens
        for b in range(self.batch):
            self.host_res_len[b] += 1
        for b in flushing:
            self.host_pages[b].append(self.host_new_page[b])
            self.host_res_len[b] = 0
        assert all(r < P for r in self.host_res_len)

    def append(self, k_new, v_new, stream=None):
        kb.append_token(self.cfg, k_new, v_new, self.res_k, self.res_v, self.res_len, self.err, stream)

    def flush(self, stream=None):
        kb.flush_residual(self.cfg, self.res_k, self.res_v, self.res_len, self.new_page, self.page_table,
                          self.num_pages, self.pool, self.err, stream)

    def append_flush(self, k_new, v_new, stream=None):
        """append then flush, in one launch."""
        kb.append_flush(self.cfg, k_new, v_new, self.res_k, self.res_v, self.res_len, self.new_page,
                        self.page_table, self.num_pages, self.pool, self.counters, self.err, stream)

    def attend(self, q, out, sm_scale=None, stream=None):
        kb.decode_attention(self.cfg, self.pool, q, self.page_table, self.num_pages, self.res_k, self.res_v,
                            self.res_len, out, self.workspace, sm_scale, self.err, stream)

    def step(self, q, k_new, v_new, out, sm_scale=None, stream=None):
        """One decode step: append, flush full windows, attend.  The host tracks every
        window's length, so the flush (quantize of the full windows and the page-table
        commit) is launched only on steps where some window fills: once every P steps
        per sequence.  Append, flush and commit stay separate launches: the single
        append_flush launch needs 41 KB of shared memory per CTA and, chained before the
        decode, delays the decode's CTAs more than it saves (measured on B200: 40.1 vs
        34.3 us per layer of the 8B-shaped 32-layer step)."""
        flushing = self.reserve_flush_pages()
        self.append(k_new, v_new, stream)
        if flushing:
            self.flush(stream)
        self.attend(q, out, sm_scale, stream)
        self.commit_host(flushing)

    def record(self, page: int, head: int) -> torch.Tensor:
        """Bytes of record (page, head) (a view into the pool)."""
        H, R = self.cfg.num_kv_heads, self.record_bytes
        off = (page * H + head) * R
        return self.pool[off:off + R]

    def check_errors(self) -> int:
        return int(self.err.item())
