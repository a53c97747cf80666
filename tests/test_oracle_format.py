"""Pins of the oracle's page record: layout sizes, bit packing, boost selection,
the two-plane split of boosted channels and the KIVI (no boost) special case."""
import json
import os

import numpy as np
import pytest

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

F16, BF16 = oracle.F16, oracle.BF16
HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    with open(os.path.join(HERE, "golden", "packing_examples.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("row", _golden()["layout"], ids=lambda r: f"P{r['P']}k{r['k']}")
def test_layout_sizes_hand_worked(row):
    L = oracle.layout(row["P"], row["D"], row["k"], row["G"])
    assert L["payload_bytes"] == row["payload"]
    assert L["record_bytes"] == row["record"]
    order = ["k_codes", "kb_codes", "v_codes", "k_scale", "k_zero", "kb_scale", "v_scale",
             "v_zero", "boost_idx"]
    offs = [L[n] for n in order]
    assert offs == sorted(offs) and offs[0] == 0
    assert all(o % 16 == 0 for o in offs[:-1])


def _page_with_codes(word_codes, cfg):
    """A page whose token 0 / channels 0..15 plane-A codes are word_codes and whose
    other channels are constant, with no boost (k = 0) so codes are plain 2-bit."""
    P, D = cfg.P, cfg.D
    K = np.zeros((P, D), np.float32)
    # channel c: token 0 carries code*1.0, the group spans [0, 3] (token 1 = 3, token 2 = 0)
    for c in range(16):
        K[0, c] = word_codes[c]
        K[1, c] = 3.0
        K[2, c] = 0.0
    return syn.to_bits(K, cfg.dtype), syn.to_bits(np.zeros((P, D), np.float32), cfg.dtype)


@pytest.mark.parametrize("case", _golden()["words"], ids=lambda c: c["word"])
def test_plane_a_word_packing_hand_worked(case):
    cfg = oracle.Cfg(P=32, k=0, Hq=1, Hkv=1)
    K, V = _page_with_codes(case["codes"], cfg)
    rec = oracle.quantize_page(K, V, cfg)
    L = oracle.layout(cfg.P, cfg.D, cfg.k, cfg.G)
    word = int(rec[L["k_codes"]:L["k_codes"] + 4].view(np.uint32)[0])
    assert word == int(case["word"], 16)


@pytest.mark.parametrize("case", _golden()["words"], ids=lambda c: c["word"])
def test_value_word_packing_hand_worked(case):
    """Values are packed along tokens: channel 0, tokens 0..15 form the first word."""
    cfg = oracle.Cfg(P=32, k=0)
    V = np.zeros((cfg.P, cfg.D), np.float32)
    V[:, 1] = 3.0                      # every token's range is [0, 3]: scale 1, zero 0
    V[:16, 0] = case["codes"]
    Vb = syn.to_bits(V, F16)
    rec = oracle.quantize_page(np.zeros((cfg.P, cfg.D), np.uint16), Vb, cfg)
    L = oracle.layout(cfg.P, cfg.D, cfg.k, cfg.G)
    word = int(rec[L["v_codes"]:L["v_codes"] + 4].view(np.uint32)[0])
    assert word == int(case["word"], 16)


def test_select_boost_matches_full_sort():
    rng = np.random.default_rng(5)
    for trial in range(200):
        dtype = F16 if trial % 2 == 0 else BF16
        P, D = int(rng.choice([32, 128])), 128
        k = int(rng.choice([0, 16, 32, 64, 128]))
        x = rng.standard_normal((P, D)) * np.exp(rng.standard_normal(D))
        if trial % 5 == 0:
            x = np.round(x)  # many exact ties in |x|
        xb = syn.to_bits(x, dtype)
        idx = oracle.select_boost(xb, k, dtype)
        score = np.abs(syn.from_bits(xb, dtype).astype(np.float64)).max(axis=0)
        want = sorted(sorted(range(D), key=lambda c: (-score[c], c))[:k])
        assert idx.tolist() == want


def _unpack(words, n_per_row):
    """Reads 2-bit elements through numpy bit ops (independent of the oracle's helpers)."""
    w = np.asarray(words, np.uint32)
    e = np.arange(16)
    shifts = (16 * (e & 1) + 2 * (e >> 1)).astype(np.uint32)
    return ((w[..., None] >> shifts) & 3).reshape(*w.shape[:-1], -1)[..., :n_per_row]


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("k", [0, 16, 32])
def test_two_plane_split_reconstructs_4bit_codes(dtype, k):
    """For boosted channels: hi*4 + lo equals the 4-bit code of that channel-group, plane A
    scale is 4x the 4-bit scale, plane B scale is the 4-bit scale; for the other
    channels plane A holds the 2-bit code.  Checked against quant_group directly."""
    rng = np.random.default_rng(7 + k + dtype)
    cfg = oracle.Cfg(P=128, k=k, dtype=dtype)
    sig = np.exp(rng.standard_normal(cfg.D))
    K = syn.to_bits(rng.standard_normal((cfg.P, cfg.D)) * sig, dtype)
    V = syn.to_bits(rng.standard_normal((cfg.P, cfg.D)), dtype)
    rec = oracle.quantize_page(K, V, cfg)
    L = oracle.layout(cfg.P, cfg.D, k, cfg.G)
    kA = _unpack(rec[L["k_codes"]:L["kb_codes"]].view(np.uint32).reshape(cfg.P, 8), 128)
    kB = (_unpack(rec[L["kb_codes"]:L["v_codes"]].view(np.uint32).reshape(cfg.P, k // 16), k)
          if k else np.zeros((cfg.P, 0), np.uint32))
    ks = rec[L["k_scale"]:L["k_zero"]].view(np.uint16).reshape(4, 128)
    kz = rec[L["k_zero"]:L["kb_scale"]].view(np.uint16).reshape(4, 128)
    kbs = rec[L["kb_scale"]:L["v_scale"]].view(np.uint16).reshape(4, k)
    idx = rec[L["boost_idx"]:L["boost_idx"] + k]
    assert idx.tolist() == oracle.select_boost(K, k, dtype).tolist()
    row = {int(c): j for j, c in enumerate(idx)}
    for g in range(4):
        for c in range(cfg.D):
            grp = K[g * 32:(g + 1) * 32, c]
            if c in row:
                j = row[c]
                c4, s4, z4 = oracle.quant_group(grp, 4, dtype)
                hi, lo = kA[g * 32:(g + 1) * 32, c], kB[g * 32:(g + 1) * 32, j]
                assert np.array_equal(hi * 4 + lo, c4)
                assert kbs[g, j] == s4
                assert oracle.value(int(ks[g, c]), dtype) == 4 * oracle.value(s4, dtype)
                assert kz[g, c] == z4
            else:
                c2, s2, z2 = oracle.quant_group(grp, 2, dtype)
                assert np.array_equal(kA[g * 32:(g + 1) * 32, c], c2)
                assert ks[g, c] == s2 and kz[g, c] == z2


def test_golden_4bit_split():
    for row in _golden()["split_4bit"]:
        assert row["hi"] * 4 + row["lo"] == row["code4"]
        assert row["code4"] >> 2 == row["hi"] and row["code4"] & 3 == row["lo"]


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_dequantize_page_matches_groupwise_dequant(dtype):
    """K^ from the two planes equals code4*s4 + mn (boosted) or code*s + mn (normal) and
    V^ equals per-token code*s + mn, exactly in fp64; errors stay within scale/2."""
    rng = np.random.default_rng(9 + dtype)
    cfg = oracle.Cfg(P=64, k=32, dtype=dtype)
    sig = np.exp(rng.standard_normal(cfg.D))
    sig[[3, 50, 77]] *= 15
    K = syn.to_bits(rng.standard_normal((cfg.P, cfg.D)) * sig, dtype)
    V = syn.to_bits(rng.standard_normal((cfg.P, cfg.D)), dtype)
    rec = oracle.quantize_page(K, V, cfg)
    Kh, Vh = oracle.dequantize_page(rec, cfg)
    idx = set(oracle.select_boost(K, cfg.k, dtype).tolist())
    assert {3, 50, 77} <= idx  # outlier channels are boosted
    for g in range(cfg.P // cfg.G):
        for c in range(cfg.D):
            grp = K[g * 32:(g + 1) * 32, c]
            bits = 4 if c in idx else 2
            codes, sb, zb = oracle.quant_group(grp, bits, dtype)
            want = codes * oracle.value(sb, dtype) + oracle.value(zb, dtype)
            assert np.array_equal(Kh[g * 32:(g + 1) * 32, c], want)
    for t in range(cfg.P):
        codes, sb, zb = oracle.quant_group(V[t], 2, dtype)
        assert np.array_equal(Vh[t], codes * oracle.value(sb, dtype) + oracle.value(zb, dtype))


def test_k0_is_uniform_2bit_kivi():
    rng = np.random.default_rng(11)
    cfg0 = oracle.Cfg(P=128, k=0)
    K = syn.to_bits(rng.standard_normal((128, 128)) * 5, F16)
    V = syn.to_bits(rng.standard_normal((128, 128)), F16)
    Kh, Vh = oracle.dequantize_page(oracle.quantize_page(K, V, cfg0), cfg0)
    for c in range(0, 128, 7):
        for g in range(4):
            codes, sb, zb = oracle.quant_group(K[g * 32:(g + 1) * 32, c], 2, F16)
            assert np.array_equal(Kh[g * 32:(g + 1) * 32, c],
                                  codes * oracle.value(sb, F16) + oracle.value(zb, F16))
    # boosting every channel (k = D) gives a strictly smaller key error than k = 0
    cfgD = oracle.Cfg(P=128, k=128)
    KhD, _ = oracle.dequantize_page(oracle.quantize_page(K, V, cfgD), cfgD)
    Kv = syn.from_bits(K, F16).astype(np.float64)
    assert np.abs(KhD - Kv).mean() < 0.3 * np.abs(Kh - Kv).mean()
