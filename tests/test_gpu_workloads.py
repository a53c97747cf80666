"""Full-size parity on the five seeded workloads, in the launch configuration the
benchmark times (PagedKVCache.step: append, flush, attend).

The GPU runs every sequence and every decode step of the workload.  The oracle
follows a sample of sequences through the same steps (its own quantization of the
raw inputs, its own residual bookkeeping) and is compared at sampled steps:
every record of the sampled sequences must match byte for byte, and their attention
outputs must be within the method's tolerance."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn
from bit_mixed_precision_channel_b200.cache import PagedKVCache

from _kv import assert_attention_close, kcfg, ocfg, to_dev

pytestmark = pytest.mark.gpu


def _check_steps(steps):
    s = {0, steps - 1}
    if steps > 8:
        s.add(steps // 2)
    return sorted(s)


def run_workload(w: syn.Workload, steps: int | None = None, lengths=None):
    cfg = kcfg(w)
    oc = ocfg(cfg)
    B, P = w.batch, w.P
    steps = w.steps if steps is None else steps
    lens = syn.lengths(w) if lengths is None else np.asarray(lengths)
    max_pages = int(max(lens) // P + steps // P + 2)
    pool_pages = int(sum(lens // P) + B * (steps // P + 2))
    cache = PagedKVCache(cfg, B, max_pages, pool_pages, page_order=syn.page_order(w, pool_pages))
    sigma = syn.key_channel_sigma(w)
    sampled = sorted({0, B // 2, B - 1})
    ocache = oracle.OracleCache(oc, len(sampled), pool_pages)
    for b in range(B):
        L = int(lens[b])
        K = syn.keys(w, b, 0, L, sigma)
        V = syn.values(w, b, 0, L)
        cache.prefill(b, to_dev(K, w.dtype), to_dev(V, w.dtype))
        if b in sampled:
            ocache.prefill(sampled.index(b), K, V, cache.host_pages[b])
        del K, V
    out = torch.empty(B, w.Hq, w.D, device="cuda")
    sm = 1.0 / math.sqrt(w.D)
    g = w.gqa
    checks = _check_steps(steps)
    n_checked = 0
    for s in range(steps):
        kn, vn = syn.step_tokens(w, s, sigma)
        q = syn.queries(w, s)
        cache.step(to_dev(q, w.dtype), to_dev(kn, w.dtype), to_dev(vn, w.dtype), out)
        new = cache.new_page.cpu().numpy()
        ocache.append(kn[sampled], vn[sampled])
        ocache.flush(new[sampled])
        if s in checks:
            got = out.cpu().numpy()
            for i, b in enumerate(sampled):
                for kvh in sorted({0, w.Hkv - 1}):
                    want = ocache.attend_unit(i, kvh, q[b], sm)
                    assert_attention_close(got[b, kvh * g:(kvh + 1) * g], want,
                                           f"{w.name} step {s} seq {b} kv head {kvh}")
                    n_checked += 1
    torch.cuda.synchronize()
    assert cache.err.item() == 0
    # every record of the sampled sequences, prefill and flushed pages alike
    payload = kb.page_layout(cfg)["payload_bytes"]
    recs = cache.pool.view(pool_pages, w.Hkv, -1)
    for i, b in enumerate(sampled):
        assert cache.host_pages[b] == ocache.seqs[i].pages
        pages = ocache.seqs[i].pages
        got = recs[torch.tensor(pages, device="cuda", dtype=torch.long)].cpu().numpy()[..., :payload]
        want = ocache.pool[pages][..., :payload]
        if not np.array_equal(got, want):
            bad = np.argwhere((got != want).any(axis=-1))
            raise AssertionError(f"{w.name} seq {b}: {len(bad)} records differ, first (page idx, head) {bad[0]}")
    return n_checked


@pytest.mark.parametrize("name", syn.ORDER)
def test_workload_full_size(name):
    w = syn.WORKLOADS[name]
    assert run_workload(w) > 0


def test_tiny_with_flushes():
    """250-token prompt, pages of 32: 7 pages + 26 residual tokens; over 40 steps the
    window fills and is flushed twice (steps 5 and 37) and ends holding 2 tokens."""
    w = syn.WORKLOADS["tiny"]
    assert run_workload(w, steps=40, lengths=[250]) > 0
