"""Full-size parity on the five seeded workloads, in the launch configuration the
benchmark times (PagedKVCache.step: append, flush, attend).

The GPU runs every sequence and every decode step of the workload.  Every record
the GPU wrote (prefill pages and pages flushed during the steps, of every sequence and
KV head) must equal, byte for byte, the oracle's quantization of the same raw tokens.
The oracle also follows a sample of sequences through the same steps (its own
residual bookkeeping and fp64 attention), and their attention outputs must be within
the method's tolerance at sampled steps."""
import concurrent.futures as cf
import math
import os

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


def check_all_records(w: syn.Workload, cfg, cache, lens, steps, sigma):
    """Every page of every sequence: the token stream of sequence b is its prompt followed
    by the token it appended at each step, and page i of b holds stream tokens
    [i P, (i + 1) P) whether it was written at prefill or by a flush."""
    oc = ocfg(cfg)
    P, B, H = w.P, w.batch, w.Hkv
    payload = kb.page_layout(cfg)["payload_bytes"]
    pool = cache.pool.view(cache.pool_pages, H, -1).cpu().numpy()
    step_k = np.stack([syn.step_tokens(w, s, sigma)[0] for s in range(steps)], axis=1) if steps else None
    step_v = np.stack([syn.step_tokens(w, s, sigma)[1] for s in range(steps)], axis=1) if steps else None

    def check_seq(b):
        L = int(lens[b])
        K, V = syn.keys(w, b, 0, L, sigma), syn.values(w, b, 0, L)
        if steps:
            K, V = np.concatenate([K, step_k[b]]), np.concatenate([V, step_v[b]])
        bad = []
        for i, pg in enumerate(cache.host_pages[b]):
            for h in range(H):
                want = oracle.quantize_page(K[i * P:(i + 1) * P, h], V[i * P:(i + 1) * P, h], oc)[:payload]
                if not np.array_equal(pool[pg, h, :payload], want):
                    bad.append((b, i, h))
        return len(cache.host_pages[b]) * H, bad

    with cf.ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1))) as ex:
        res = list(ex.map(check_seq, range(B)))
    n = sum(r[0] for r in res)
    bad = [x for r in res for x in r[1]]
    assert not bad, f"{w.name}: {len(bad)} of {n} records differ, first (seq, page, head) {bad[0]}"
    return n


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
    n_records = check_all_records(w, cfg, cache, lens, steps, sigma)
    assert n_records == sum(len(p) for p in cache.host_pages) * w.Hkv
    # the sampled sequences' page lists and records also agree with the oracle's bookkeeping
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
