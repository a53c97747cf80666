"""Pins of the oracle's boost options: the query-aware channel ranking (the MixKVQ
reading: channel range over the page times a query-relevance weight) and the per-head
boost count (fewer boosted channels than the record has plane-B rows).

The query-aware ranking is pinned by a hand-worked page (tests/golden), by its
reduction to the magnitude ranking when every channel's minimum is zero and every
weight is one, by permutation equivariance and by a full sort; the per-head count by
its reduction to a record laid out for exactly that many rows, read back with the
independent decoder of test_oracle_format."""
import json
import os

import numpy as np
import pytest

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

from test_oracle_format import _decode_record

F16, BF16 = oracle.F16, oracle.BF16
HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    with open(os.path.join(HERE, "golden", "boost_query_examples.json")) as f:
        return json.load(f)["examples"]


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_query_ranking_hand_worked(dtype):
    for ex in _golden():
        K = np.zeros((128, 128), np.float32)
        for t, c, v in ex["nonzero"]:
            K[t, c] = v
        w = np.full(128, ex["weight_default"], np.float32)
        for c, v in ex["weight"]:
            w[c] = v
        Kb = syn.to_bits(K, dtype)
        assert oracle.select_boost_query(Kb, 3, w, dtype).tolist() == ex["top3"]
        assert oracle.select_boost_query(Kb, 4, w, dtype).tolist() == ex["top4"]
        assert oracle.select_boost_query(Kb, 5, w, dtype).tolist() == ex["top5"]
        assert oracle.select_boost_query(Kb, 7, w, dtype).tolist() == ex["top7_with_zero_scores"]
        assert oracle.select_boost(Kb, 3, dtype).tolist() == ex["magnitude_top3"]


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_query_ranking_with_unit_weights_and_zero_minima_is_the_magnitude_ranking(dtype):
    """When every channel's minimum over the page is 0 (non-negative keys with a zero in
    every channel) the range equals max |K|, so unit weights give Kitty's ranking."""
    rng = np.random.default_rng(3)
    for trial in range(20):
        K = np.abs(rng.standard_normal((128, 128)) * np.exp(rng.standard_normal(128)))
        K[rng.integers(0, 128, 128), np.arange(128)] = 0.0
        if trial % 3 == 0:
            K = np.round(K)  # exact ties
        Kb = syn.to_bits(K, dtype)
        for n in (0, 16, 32, 128):
            assert oracle.select_boost_query(Kb, n, np.ones(128, np.float32), dtype).tolist() == \
                oracle.select_boost(Kb, n, dtype).tolist()


def test_query_ranking_is_permutation_equivariant():
    rng = np.random.default_rng(4)
    for _ in range(20):
        K = syn.to_bits(rng.standard_normal((64, 128)) * np.exp(rng.standard_normal(128)), F16)
        w = np.abs(rng.standard_normal(128)).astype(np.float32)
        perm = rng.permutation(128)
        a = oracle.select_boost_query(K, 32, w, F16)
        b = oracle.select_boost_query(np.ascontiguousarray(K[:, perm]), 32, w[perm], F16)
        # channel perm[i] of the original is channel i of the permuted page; scores are
        # distinct with probability 1 here, so ties do not reorder
        assert sorted(perm[b].tolist()) == a.tolist()


def test_query_ranking_matches_full_sort():
    rng = np.random.default_rng(5)
    for trial in range(100):
        dtype = F16 if trial % 2 == 0 else BF16
        K = rng.standard_normal((128, 128)) * np.exp(rng.standard_normal(128))
        if trial % 4 == 0:
            K = np.round(K)
        Kb = syn.to_bits(K, dtype)
        Kv = syn.from_bits(Kb, dtype).astype(np.float32)
        w = np.abs(rng.standard_normal(128)).astype(np.float32)
        if trial % 5 == 0:
            w = np.round(w * 4) / 4  # repeated weights, exact ties in the score
        rng_c = (Kv.max(axis=0) - Kv.min(axis=0)).astype(np.float32)
        score = (w * rng_c).astype(np.float32)
        n = int(rng.choice([0, 16, 32, 64, 128]))
        want = sorted(sorted(range(128), key=lambda c: (-float(score[c]), c))[:n])
        assert oracle.select_boost_query(Kb, n, w, dtype).tolist() == want


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("k,n", [(32, 32), (32, 16), (32, 0), (64, 48), (128, 16)])
def test_per_head_boost_count_reduces_to_a_narrower_record(dtype, k, n):
    """n of k rows used: the keys decode exactly as a record laid out for n rows (the
    same boosted channels, codes and scales); the unused plane-B rows, their scales and
    their indices are zero; the values are untouched."""
    rng = np.random.default_rng(7 + k + n + dtype)
    sig = np.exp(rng.standard_normal(128))
    K = syn.to_bits(rng.standard_normal((128, 128)) * sig, dtype)
    V = syn.to_bits(rng.standard_normal((128, 128)), dtype)
    rec = oracle.quantize_page_ex(K, V, oracle.Cfg(P=128, k=k, dtype=dtype), n_boost=n)
    if n == k:
        assert np.array_equal(rec, oracle.quantize_page(K, V, oracle.Cfg(P=128, k=k, dtype=dtype)))
    narrow_cfg = oracle.Cfg(P=128, k=n, dtype=dtype)
    narrow = oracle.quantize_page(K, V, narrow_cfg)
    d, e = _decode_record(rec, 128, k, dtype), _decode_record(narrow, 128, n, dtype)
    assert d["idx"][:n].tolist() == e["idx"].tolist() and not d["idx"][n:].any()
    assert np.array_equal(d["kA"], e["kA"]) and np.array_equal(d["ks"], e["ks"]) and np.array_equal(d["kz"], e["kz"])
    assert np.array_equal(d["kB"][:, :n], e["kB"]) and not d["kB"][:, n:].any()
    assert np.array_equal(d["kbs"][:, :n], e["kbs"]) and not d["kbs"][:, n:].any()
    assert np.array_equal(d["v"], e["v"]) and np.array_equal(d["vs"], e["vs"]) and np.array_equal(d["vz"], e["vz"])
    Kw, _ = oracle.dequantize_page(rec, oracle.Cfg(P=128, k=k, dtype=dtype))
    Kn, _ = oracle.dequantize_page(narrow, narrow_cfg)
    assert np.array_equal(Kw, Kn)


def test_query_aware_record_boosts_the_query_ranked_channels():
    """The query-aware record's boosted channels are select_boost_query's, and their keys
    decode as 4-bit codes (hi * 4 + lo) of the same groups."""
    rng = np.random.default_rng(11)
    cfg = oracle.Cfg(P=128, k=32)
    K = syn.to_bits(rng.standard_normal((128, 128)) * np.exp(rng.standard_normal(128)), F16)
    V = syn.to_bits(rng.standard_normal((128, 128)), F16)
    w = np.abs(rng.standard_normal(128)).astype(np.float32) * 3
    d = _decode_record(oracle.quantize_page_ex(K, V, cfg, weight=w), 128, 32, F16)
    idx = oracle.select_boost_query(K, 32, w, F16)
    assert d["idx"].tolist() == idx.tolist()
    assert idx.tolist() != oracle.select_boost(K, 32, F16).tolist()  # a different set than magnitude
    for j, c in enumerate(idx):
        for g in range(4):
            c4, s4, z4 = oracle.quant_group(K[g * 32:(g + 1) * 32, c], 4, F16)
            assert np.array_equal(d["kA"][g * 32:(g + 1) * 32, c] * 4 + d["kB"][g * 32:(g + 1) * 32, j], c4)
            assert d["kbs"][g, j] == s4
