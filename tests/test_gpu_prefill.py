"""GPU parity of the MiniKV prefill path: causal prefill attention with
cumulative attention scores, heavy-hitter + recent-window retention, the gather of the
kept tokens and their quantization.

Outputs are within the method's tolerance of the oracle's fp64 attention; scores within
|d| <= 2e-3 + 1e-3 * score of the oracle's fp64 scores; the retention decision, an
integer result decided by floating point, is compared with the oracle's rule applied to
the kernel's own fp32 scores (both sides decide in the same precision); the kept tokens
and their records are compared byte for byte."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn

from _kv import assert_attention_close, ocfg, to_dev

pytestmark = pytest.mark.gpu


def _inputs(rng, L, Hq, Hkv, dtype):
    sig = np.exp(rng.standard_normal((Hkv, 128))).astype(np.float32)
    Q = syn.to_bits(rng.standard_normal((L, Hq, 128)).astype(np.float32), dtype)
    K = syn.to_bits(rng.standard_normal((L, Hkv, 128)).astype(np.float32) * sig, dtype)
    V = syn.to_bits(rng.standard_normal((L, Hkv, 128)).astype(np.float32), dtype)
    return Q, K, V


def _prefill(cfg, Q, K, V):
    dt = cfg.dtype
    L = Q.shape[0]
    out = torch.full((L, cfg.num_q_heads, 128), float("nan"), device="cuda")
    scores = torch.full((cfg.num_kv_heads, L), float("nan"), device="cuda")
    ws = torch.zeros(max(kb.prefill_workspace_bytes(cfg, L), 256), dtype=torch.uint8, device="cuda")
    kb.prefill_attention(cfg, to_dev(Q, dt), to_dev(K, dt), to_dev(V, dt), out, scores, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), scores.cpu().numpy()


@pytest.mark.parametrize("L,gqa,Hkv,dtype", [
    (300, 4, 2, kb.F16), (1000, 4, 1, kb.BF16), (64, 1, 1, kb.F16), (1, 2, 1, kb.F16), (257, 8, 1, kb.BF16),
    (129, 2, 2, kb.F16),
])
def test_prefill_output_and_scores_match_oracle(L, gqa, Hkv, dtype):
    rng = np.random.default_rng(L + gqa + dtype)
    cfg = kb.Config(num_q_heads=gqa * Hkv, num_kv_heads=Hkv, page_tokens=128, num_boost=32, dtype=dtype)
    Q, K, V = _inputs(rng, L, gqa * Hkv, Hkv, dtype)
    out, scores = _prefill(cfg, Q, K, V)
    O, A = oracle.prefill_attention(Q, K, V, dtype, 1.0 / math.sqrt(128))
    assert_attention_close(out, O, f"prefill L{L}")
    err = np.abs(scores - A)
    assert (err <= 2e-3 + 1e-3 * A).all(), f"scores: max abs {err.max():.2e}"


def test_long_prefill_scores_sum_to_the_query_count():
    """L = 4096, 32 / 8 heads (the oracle's fp64 attention would take minutes): every
    query row's probabilities sum to one, so each KV head's scores sum to gqa * L, and the
    output rows are finite."""
    rng = np.random.default_rng(2)
    L, Hq, Hkv = 4096, 32, 8
    cfg = kb.Config(num_q_heads=Hq, num_kv_heads=Hkv, page_tokens=128, num_boost=32)
    Q, K, V = _inputs(rng, L, Hq, Hkv, kb.F16)
    out, scores = _prefill(cfg, Q, K, V)
    assert np.isfinite(out).all() and (scores >= 0).all()
    assert np.allclose(scores.astype(np.float64).sum(axis=1), 4 * L, rtol=2e-4)
    # the first positions collect the most attention in a causal prefill of random data
    assert (scores[:, :16].mean(axis=1) > scores[:, -16:].mean(axis=1)).all()


@pytest.mark.parametrize("nh,nr", [(0, 0), (0, 5), (7, 0), (25, 25), (40, 30), (100, 100), (3, 200)])
def test_retention_matches_oracle_rule_on_given_scores(nh, nr):
    """Scores with many exact ties (quarter steps): the kept positions equal the oracle's."""
    rng = np.random.default_rng(nh * 7 + nr)
    H, L = 3, 150
    cfg = kb.Config(num_q_heads=H, num_kv_heads=H, page_tokens=128, num_boost=32)
    s = (np.round(rng.random((H, L)) * 8) / 4).astype(np.float32)
    keep = torch.full((H, L), -1, dtype=torch.int32, device="cuda")
    n_keep = torch.zeros(H, dtype=torch.int32, device="cuda")
    kb.retain_tokens(cfg, torch.from_numpy(s).cuda(), nh, nr, keep, n_keep)
    torch.cuda.synchronize()
    for h in range(H):
        want = oracle.retain(s[h].astype(np.float64), nh, nr)
        assert n_keep[h].item() == len(want)
        assert keep[h, :len(want)].tolist() == want.tolist()


@pytest.mark.parametrize("dtype", [kb.F16, kb.BF16])
def test_prefill_retain_gather_quantize_pipeline(dtype):
    """The whole path: prefill attention, 25% heavy hitters + 25% recent tokens, gather,
    then page quantization of the kept tokens; records byte-exact against the oracle's
    quantization of the same kept tokens."""
    rng = np.random.default_rng(40 + dtype)
    L, Hq, Hkv, P = 512, 8, 2, 64
    cfg = kb.Config(num_q_heads=Hq, num_kv_heads=Hkv, page_tokens=P, num_boost=16, dtype=dtype)
    Q, K, V = _inputs(rng, L, Hq, Hkv, dtype)
    out, scores = _prefill(cfg, Q, K, V)
    nh = nr = L // 4
    keep = torch.full((Hkv, L), -1, dtype=torch.int32, device="cuda")
    n_keep = torch.zeros(Hkv, dtype=torch.int32, device="cuda")
    kb.retain_tokens(cfg, torch.from_numpy(scores).cuda(), nh, nr, keep, n_keep)
    n = nh + nr
    k_out = torch.empty(n, Hkv, 128, dtype=kb.torch_dtype(dtype), device="cuda")
    v_out = torch.empty_like(k_out)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb.gather_tokens(cfg, to_dev(K, dtype), to_dev(V, dtype), keep, n, k_out, v_out, err)
    n_pages = n // P
    pool = torch.zeros(n_pages * Hkv * kb.page_bytes(cfg), dtype=torch.uint8, device="cuda")
    kb.quantize_pages(cfg, kb.Source.token_major(k_out, cfg), kb.Source.token_major(v_out, cfg),
                      torch.arange(n_pages, dtype=torch.int32, device="cuda"), pool, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    kept = keep.cpu().numpy()[:, :n]
    oc = ocfg(cfg)
    recs = pool.cpu().numpy().reshape(n_pages, Hkv, -1)
    payload = kb.page_layout(cfg)["payload_bytes"]
    for h in range(Hkv):
        assert kept[h].tolist() == oracle.retain(scores[h].astype(np.float64), nh, nr).tolist()
        Kh, Vh = K[kept[h], h], V[kept[h], h]
        got_k = k_out[:, h].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got_k, Kh)
        for i in range(n_pages):
            want = oracle.quantize_page(Kh[i * P:(i + 1) * P], Vh[i * P:(i + 1) * P], oc)
            assert np.array_equal(recs[i, h, :payload], want[:payload]), (h, i)
