"""Pins of the oracle's decode attention and of its host-side pipeline (CPU only).

decode_unit is checked against torch's fp64 scaled_dot_product_attention on the
dequantized tokens (a library routine), against closed forms (identical keys give the
mean of the values; one dominant key gives its value) and against invariances (page
order, empty sequence).  The pipeline is checked against the prefill/append/flush
rules stated in its docstring."""
import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

F16, BF16 = oracle.F16, oracle.BF16


def _pool_from_pages(cfg, pages_kv):
    pool = np.zeros((len(pages_kv), cfg.Hkv, cfg.record_bytes), np.uint8)
    for p, (K, V) in enumerate(pages_kv):
        for h in range(cfg.Hkv):
            pool[p, h] = oracle.quantize_page(K[:, h], V[:, h], cfg)
    return pool


def _sdpa(q, K, V, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        scale=scale)
    return out[0].numpy()


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("gqa", [1, 4])
def test_decode_unit_matches_torch_sdpa(dtype, gqa):
    rng = np.random.default_rng(3 + gqa + dtype)
    cfg = oracle.Cfg(P=32, k=16, Hq=2 * gqa, Hkv=2, dtype=dtype)
    n_pages, res_len = 3, 11
    pages = []
    for _ in range(n_pages):
        K = syn.to_bits(rng.standard_normal((cfg.P, cfg.Hkv, cfg.D)) * 3, dtype)
        V = syn.to_bits(rng.standard_normal((cfg.P, cfg.Hkv, cfg.D)), dtype)
        pages.append((K, V))
    pool = _pool_from_pages(cfg, pages)
    order = [2, 0, 1]
    rk = syn.to_bits(rng.standard_normal((res_len, cfg.D)), dtype)
    rv = syn.to_bits(rng.standard_normal((res_len, cfg.D)), dtype)
    q = syn.to_bits(rng.standard_normal((gqa, cfg.D)), dtype)
    head = 1
    sm = 1 / np.sqrt(cfg.D)
    out = oracle.decode_unit(pool, cfg, head, order, rk, rv, q, sm)
    Ks, Vs = [], []
    for p in order:
        Kh, Vh = oracle.dequantize_page(pool[p, head], cfg)
        Ks.append(Kh)
        Vs.append(Vh)
    Ks.append(oracle.values(rk, dtype))
    Vs.append(oracle.values(rv, dtype))
    want = _sdpa(oracle.values(q, dtype), np.concatenate(Ks), np.concatenate(Vs), sm)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_identical_keys_give_mean_of_values():
    cfg = oracle.Cfg(P=32, k=16)
    rng = np.random.default_rng(4)
    k_row = syn.to_bits(rng.standard_normal(cfg.D), F16)
    K = np.broadcast_to(k_row, (cfg.P, 1, cfg.D)).copy()
    V = syn.to_bits(rng.standard_normal((cfg.P, 1, cfg.D)), F16)
    pool = _pool_from_pages(cfg, [(K, V), (K, V)])
    q = syn.to_bits(rng.standard_normal((1, cfg.D)), F16)
    out = oracle.decode_unit(pool, cfg, 0, [0, 1], np.zeros((0, cfg.D), np.uint16),
                             np.zeros((0, cfg.D), np.uint16), q, 0.1)
    _, Vh = oracle.dequantize_page(pool[0, 0], cfg)
    np.testing.assert_allclose(out[0], Vh.mean(axis=0), rtol=0, atol=1e-13)


def test_dominant_key_gives_its_value():
    cfg = oracle.Cfg(P=32, k=16)
    rng = np.random.default_rng(6)
    K = np.zeros((cfg.P, 1, cfg.D), np.float32)
    K[:, 0, :] = rng.standard_normal((cfg.P, cfg.D)) * 0.01
    K[17, 0, :] = 8.0
    V = rng.standard_normal((cfg.P, 1, cfg.D))
    Kb, Vb = syn.to_bits(K, F16), syn.to_bits(V, F16)
    pool = _pool_from_pages(cfg, [(Kb, Vb)])
    q = syn.to_bits(np.full((1, cfg.D), 4.0), F16)
    out = oracle.decode_unit(pool, cfg, 0, [0], np.zeros((0, cfg.D), np.uint16),
                             np.zeros((0, cfg.D), np.uint16), q, 1.0)
    _, Vh = oracle.dequantize_page(pool[0, 0], cfg)
    np.testing.assert_allclose(out[0], Vh[17], rtol=0, atol=1e-12)


def test_residual_only_is_exact_attention_on_inputs():
    cfg = oracle.Cfg(P=32, k=16)
    rng = np.random.default_rng(8)
    rk = syn.to_bits(rng.standard_normal((7, cfg.D)), F16)
    rv = syn.to_bits(rng.standard_normal((7, cfg.D)), F16)
    q = syn.to_bits(rng.standard_normal((1, cfg.D)), F16)
    pool = np.zeros((1, 1, cfg.record_bytes), np.uint8)
    out = oracle.decode_unit(pool, cfg, 0, [], rk, rv, q, 0.3)
    want = _sdpa(oracle.values(q, F16), oracle.values(rk, F16), oracle.values(rv, F16), 0.3)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


def test_empty_sequence_gives_zero():
    cfg = oracle.Cfg(P=32, k=16)
    pool = np.zeros((1, 1, cfg.record_bytes), np.uint8)
    out = oracle.decode_unit(pool, cfg, 0, [], np.zeros((0, cfg.D), np.uint16),
                             np.zeros((0, cfg.D), np.uint16), np.zeros((1, cfg.D), np.uint16), 1.0)
    assert (out == 0).all()


def test_pipeline_prefill_append_flush_rules():
    w = syn.WORKLOADS["tiny"]
    cfg = oracle.Cfg(D=w.D, Hq=w.Hq, Hkv=w.Hkv, P=w.P, G=w.G, k=w.k, dtype=w.dtype)
    L = 250
    K = syn.keys(w, 0, 0, L)
    V = syn.values(w, 0, 0, L)
    cache = oracle.OracleCache(cfg, batch=1, pool_pages=32)
    n_full = L // cfg.P
    cache.prefill(0, K, V, list(range(10, 10 + n_full)))
    assert cache.seqs[0].pages == list(range(10, 10 + n_full))
    assert cache.res_len(0) == L % cfg.P
    # the quantized pages are exactly quantize_page of their token ranges
    for i in range(n_full):
        rec = oracle.quantize_page(K[i * 32:(i + 1) * 32, 0], V[i * 32:(i + 1) * 32, 0], cfg)
        assert np.array_equal(cache.pool[10 + i, 0], rec)
    # append until the window is full, then flush into page 3
    steps = cfg.P - L % cfg.P
    for s in range(steps):
        kn, vn = syn.step_tokens(w, s)
        cache.append(kn, vn)
    assert cache.res_len(0) == cfg.P
    assert cache.flush([3]) == [0]
    assert cache.res_len(0) == 0 and cache.seqs[0].pages[-1] == 3
    window_k = np.concatenate([K[n_full * 32:, 0]] + [syn.step_tokens(w, s)[0][0] for s in range(steps)])
    window_v = np.concatenate([V[n_full * 32:, 0]] + [syn.step_tokens(w, s)[1][0] for s in range(steps)])
    assert np.array_equal(cache.pool[3, 0], oracle.quantize_page(window_k, window_v, cfg))
    # attention of the cache equals decode_unit over the same token list
    q = syn.queries(w, 0)
    out = cache.attend(q, 1 / np.sqrt(cfg.D))
    direct = oracle.decode_unit(cache.pool, cfg, 0, cache.seqs[0].pages, np.zeros((0, 128), np.uint16),
                                np.zeros((0, 128), np.uint16), q[0], 1 / np.sqrt(cfg.D))
    np.testing.assert_array_equal(out[0], direct)


def test_page_table_order_only_permutes_tokens():
    """Attention is a sum over tokens: listing the same pages in another order changes
    the result only by fp64 rounding."""
    rng = np.random.default_rng(12)
    cfg = oracle.Cfg(P=32, k=16)
    pages = [(syn.to_bits(rng.standard_normal((32, 1, 128)) * 2, F16),
              syn.to_bits(rng.standard_normal((32, 1, 128)), F16)) for _ in range(4)]
    pool = _pool_from_pages(cfg, pages)
    q = syn.to_bits(rng.standard_normal((1, 128)), F16)
    e = np.zeros((0, 128), np.uint16)
    a = oracle.decode_unit(pool, cfg, 0, [0, 1, 2, 3], e, e, q, 0.2)
    b = oracle.decode_unit(pool, cfg, 0, [3, 1, 0, 2], e, e, q, 0.2)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def _grid_page(rng, P, k, G=32):
    """One page [P][D] whose every key group and value row sits exactly on its own
    quantization grid.  Keys of k channels span 15 steps of 1/8, 1/4 or 1/2 (a 4-bit
    grid) with magnitudes of at least 1, the others span 3 steps of 1/16 or 1/8 (a
    2-bit grid) below 0.4, so the magnitude ranking boosts exactly the k wide channels;
    every value row spans 3 steps of 1/4, 1/2 or 1.  The step is drawn per group, so a
    scale read from the wrong row or group changes the result.  All values are
    multiples of 1/16 below 8: exact in fp16 and bf16."""
    D = 128
    wide = set(rng.choice(D, size=k, replace=False).tolist())
    K = np.zeros((P, D))
    for c in range(D):
        for g in range(P // G):
            if c in wide:
                qmax, step, lo = 15, rng.choice([0.125, 0.25, 0.5]), 4
            else:
                qmax, step, lo = 3, rng.choice([0.0625, 0.125]), 0
            codes = rng.integers(0, qmax + 1, G)
            codes[rng.choice(G, 2, replace=False)] = [0, qmax]  # both ends: scale is exactly `step`
            mn = -step * rng.integers(lo, lo + 4)
            K[g * G:(g + 1) * G, c] = mn + codes * step
    V = np.zeros((P, D))
    for t in range(P):
        step = rng.choice([0.25, 0.5, 1.0])
        codes = rng.integers(0, 4, D)
        codes[rng.choice(D, 2, replace=False)] = [0, 3]
        V[t] = -step * rng.integers(0, 4) + step * codes
    return K, V


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("P,k", [(32, 0), (32, 16), (128, 32), (128, 128)])
def test_grid_exact_pages_give_exact_attention_on_the_inputs(dtype, P, k):
    """Keys on a 2/4-bit grid and values on a 2-bit grid are reproduced exactly by the
    quantizer (grid recovery), so attention over the quantized pages plus an fp16
    residual must equal exact attention over the raw inputs, here torch's fp64 SDPA,
    to fp64 rounding.  No oracle dequantizer is involved on the expected side: a
    plane, scale, zero, boost row or token-order mistake anywhere between the record
    and the softmax shows up.  k = D is the all-channels 4-bit case, k = 0 plain
    uniform 2 bits."""
    rng = np.random.default_rng(50 + P + k + dtype)
    cfg = oracle.Cfg(P=P, k=k, Hq=4, Hkv=2, dtype=dtype)
    n_pages, res_len = 3, 5
    pool = np.zeros((n_pages, cfg.Hkv, cfg.record_bytes), np.uint8)
    raw = {}
    for p in range(n_pages):
        for h in range(cfg.Hkv):
            K, V = _grid_page(rng, P, k)
            Kb, Vb = syn.to_bits(K, dtype), syn.to_bits(V, dtype)
            assert np.array_equal(oracle.values(Kb, dtype), K) and np.array_equal(oracle.values(Vb, dtype), V)
            pool[p, h] = oracle.quantize_page(Kb, Vb, cfg)
            raw[p, h] = (K, V)
    order = [1, 2, 0]
    sm = 1 / np.sqrt(cfg.D)
    for h in range(cfg.Hkv):
        rk = syn.to_bits(rng.standard_normal((res_len, cfg.D)), dtype)
        rv = syn.to_bits(rng.standard_normal((res_len, cfg.D)), dtype)
        q = syn.to_bits(rng.standard_normal((cfg.gqa, cfg.D)), dtype)
        out = oracle.decode_unit(pool, cfg, h, order, rk, rv, q, sm)
        Ks = np.concatenate([raw[p, h][0] for p in order] + [oracle.values(rk, dtype)])
        Vs = np.concatenate([raw[p, h][1] for p in order] + [oracle.values(rv, dtype)])
        want = _sdpa(oracle.values(q, dtype), Ks, Vs, sm)
        np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)
