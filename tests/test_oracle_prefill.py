"""Pins of the oracle's prefill attention with cumulative attention scores and of its
token retention (the MiniKV reading: heavy hitters by cumulative score plus a recent
window).  The output is checked against torch's scaled-dot-product attention in fp64;
the scores against the dense attention matrix on tiny inputs, their row-sum invariant,
the closed form for identical keys and a dominant key; retention against hand-worked
cases and a full sort."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

F16, BF16 = oracle.F16, oracle.BF16
HERE = os.path.dirname(os.path.abspath(__file__))


def _qkv(rng, L, Hq, Hkv, dtype, scale=1.0):
    D = 128
    Q = syn.to_bits(rng.standard_normal((L, Hq, D)) * scale, dtype)
    K = syn.to_bits(rng.standard_normal((L, Hkv, D)), dtype)
    V = syn.to_bits(rng.standard_normal((L, Hkv, D)), dtype)
    return Q, K, V


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("L,Hq,Hkv", [(1, 1, 1), (7, 4, 2), (33, 8, 1), (20, 2, 2)])
def test_prefill_output_matches_torch_causal_sdpa(dtype, L, Hq, Hkv):
    rng = np.random.default_rng(L * 10 + Hq + dtype)
    Q, K, V = _qkv(rng, L, Hq, Hkv, dtype)
    sm = 1.0 / math.sqrt(128)
    O, _ = oracle.prefill_attention(Q, K, V, dtype, sm)
    q = torch.from_numpy(syn.from_bits(Q, dtype).astype(np.float64)).permute(1, 0, 2)
    k = torch.from_numpy(syn.from_bits(K, dtype).astype(np.float64)).permute(1, 0, 2)
    v = torch.from_numpy(syn.from_bits(V, dtype).astype(np.float64)).permute(1, 0, 2)
    g = Hq // Hkv
    k, v = k.repeat_interleave(g, dim=0), v.repeat_interleave(g, dim=0)
    want = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True,
                                                           scale=sm)[0].permute(1, 0, 2).numpy()
    assert np.abs(O - want).max() < 1e-12


@pytest.mark.parametrize("L,Hq,Hkv", [(9, 4, 2), (16, 2, 1), (5, 1, 1)])
def test_cumulative_scores_are_column_sums_of_the_dense_matrix(L, Hq, Hkv):
    rng = np.random.default_rng(L + 100 * Hq)
    Q, K, V = _qkv(rng, L, Hq, Hkv, F16, scale=2.0)
    sm = 1.0 / math.sqrt(128)
    _, A = oracle.prefill_attention(Q, K, V, F16, sm)
    q = syn.from_bits(Q, F16).astype(np.float64)
    k = syn.from_bits(K, F16).astype(np.float64)
    g = Hq // Hkv
    want = np.zeros((Hkv, L))
    for h in range(Hq):
        S = q[:, h] @ k[:, h // g].T * sm
        S[np.triu_indices(L, 1)] = -np.inf
        Pm = np.exp(S - S.max(axis=1, keepdims=True))
        Pm /= Pm.sum(axis=1, keepdims=True)
        want[h // g] += Pm.sum(axis=0)
    assert np.abs(A - want).max() < 1e-12
    assert np.allclose(A.sum(axis=1), g * L, rtol=0, atol=1e-10)  # every row of P sums to one


def test_identical_keys_give_the_harmonic_tail():
    """All keys equal: row i spreads 1 / (i + 1) over positions 0..i, so token j
    receives sum_{i >= j} 1 / (i + 1) from each query head."""
    rng = np.random.default_rng(3)
    L, Hq, Hkv = 24, 4, 2
    Q, _, V = _qkv(rng, L, Hq, Hkv, F16)
    K = np.repeat(syn.to_bits(rng.standard_normal((1, Hkv, 128)), F16), L, axis=0)
    _, A = oracle.prefill_attention(Q, K, V, F16, 1.0 / math.sqrt(128))
    tail = np.array([sum(1.0 / (i + 1) for i in range(j, L)) for j in range(L)])
    assert np.abs(A - 2 * tail[None]).max() < 1e-12


def test_dominant_first_key_collects_all_attention():
    L = 16
    Q = syn.to_bits(np.ones((L, 1, 128)), F16)
    K = syn.to_bits(np.concatenate([np.full((1, 1, 128), 8.0), np.zeros((L - 1, 1, 128))]), F16)
    V = syn.to_bits(np.zeros((L, 1, 128)), F16)
    _, A = oracle.prefill_attention(Q, K, V, F16, 1.0)
    assert A[0, 0] > L - 1e-6 and A[0, 1:].max() < 1e-6


def test_output_is_causal():
    rng = np.random.default_rng(9)
    Q, K, V = _qkv(rng, 12, 2, 1, F16)
    O1, _ = oracle.prefill_attention(Q, K, V, F16, 0.1)
    K2, V2 = K.copy(), V.copy()
    K2[-1] = syn.to_bits(rng.standard_normal((1, 128)) * 5, F16)
    V2[-1] = syn.to_bits(rng.standard_normal((1, 128)) * 5, F16)
    O2, _ = oracle.prefill_attention(Q, K2, V2, F16, 0.1)
    assert np.array_equal(O1[:-1], O2[:-1]) and not np.array_equal(O1[-1], O2[-1])


def test_retention_hand_worked():
    with open(os.path.join(HERE, "golden", "retention_examples.json")) as f:
        g = json.load(f)
    a = np.array(g["scores"], np.float64)
    for c in g["cases"]:
        assert oracle.retain(a, c["n_heavy"], c["n_recent"]).tolist() == c["keep"]


def test_retention_matches_full_sort():
    rng = np.random.default_rng(12)
    for trial in range(200):
        L = int(rng.integers(1, 200))
        a = rng.random(L)
        if trial % 3 == 0:
            a = np.round(a * 4) / 4  # ties
        nh, nr = int(rng.integers(0, L + 2)), int(rng.integers(0, L + 2))
        cut = L - min(nr, L)
        heavy = sorted(range(cut), key=lambda j: (-a[j], j))[:nh]
        want = sorted(set(heavy) | set(range(cut, L)))
        assert oracle.retain(a, nh, nr).tolist() == want
