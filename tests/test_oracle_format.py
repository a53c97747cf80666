"""Pins of the oracle's page record: layout sizes, element and channel/token storage
order (hand-worked golden values), boost selection, the two-plane split of boosted
channels and the KIVI (no boost) special case.

The decoder `_decode_record` below reads a record with numpy bit operations written
from the rules stated in tests/golden/packing_examples.json, independently of the
oracle's C code."""
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


# -------------------------------------------------------------- independent decoder

def _shift(e):
    """element e = 8a + 2b + f of a word sits at bit 8b + 4f + 2a"""
    e = np.asarray(e)
    return 8 * ((e >> 1) & 3) + 4 * (e & 1) + 2 * (e >> 3)


def _key_channel(p):
    """inverse of the key storage order: position 32q + 4s + 2r + f -> channel 16s + 8r + 2q + f"""
    p = np.asarray(p)
    q, s, r, f = p >> 5, (p >> 2) & 7, (p >> 1) & 1, p & 1
    return 16 * s + 8 * r + 2 * q + f


def _boost_row(p, KB):
    p = np.asarray(p)
    q, rem = p // (4 * KB), p % (4 * KB)
    s, r, f = rem >> 2, (rem >> 1) & 1, rem & 1
    return 16 * s + 8 * r + 2 * q + f


def _key_meta_channel(p):
    """inverse of the scale/zero order: position 32i + 8q + 4j + 2r + f -> channel 16(2i + j) + 8r + 2q + f"""
    p = np.asarray(p)
    i, q, j, r, f = p >> 5, (p >> 3) & 3, (p >> 2) & 1, (p >> 1) & 1, p & 1
    return 16 * (2 * i + j) + 8 * r + 2 * q + f


def _value_token_channel(slot):
    """inverse of the value-code order: slot 16*word + element -> (token, channel), with
    word = ((2g + n) * 32 + 4w + q) * 4 + mm, element = 8a + 2(2u + v) + f,
    token 32g + 16a + 8u + 2q + f, channel 16(4n + mm) + 8v + w"""
    slot = np.asarray(slot)
    word, e = slot >> 4, slot & 15
    mm, lane, blk = word & 3, (word >> 2) & 31, word >> 7
    g, n = blk >> 1, blk & 1
    w, q = lane >> 2, lane & 3
    a, b, f = e >> 3, (e >> 1) & 3, e & 1
    u, v = b >> 1, b & 1
    return 32 * g + 16 * a + 8 * u + 2 * q + f, 16 * (4 * n + mm) + 8 * v + w


def _value_meta_token(p):
    """inverse of the value scale/zero order: position 32g + 4w + u -> token 32g + 8u + w"""
    p = np.asarray(p)
    g, w, u = p >> 5, (p >> 2) & 7, p & 3
    return 32 * g + 8 * u + w


def _words_to_positions(words):
    """[rows][n_words] uint32 -> [rows][16 * n_words] codes by storage position"""
    w = np.asarray(words, np.uint32)
    e = np.arange(16)
    return ((w[..., None] >> _shift(e).astype(np.uint32)) & 3).reshape(w.shape[0], -1)


def _decode_record(rec, P, k, dtype):
    """-> dict of planes in natural order: kA [P][128], kB [P][k], v [P][128], scales..."""
    L = oracle.layout(P, 128, k, 32)
    KB = k // 16
    u16 = lambda a, b: rec[a:b].view(np.uint16)
    kA_pos = _words_to_positions(rec[L["k_codes"]:L["kb_codes"]].view(np.uint32).reshape(P, 8))
    kA = np.zeros((P, 128), np.int64)
    kA[:, _key_channel(np.arange(128))] = kA_pos
    kB = np.zeros((P, k), np.int64)
    if k:
        kB_pos = _words_to_positions(rec[L["kb_codes"]:L["v_codes"]].view(np.uint32).reshape(P, KB))
        kB[:, _boost_row(np.arange(k), KB)] = kB_pos
    v_slots = _words_to_positions(rec[L["v_codes"]:L["k_scale"]].view(np.uint32)[None, :])[0]
    v = np.zeros((P, 128), np.int64)
    tok, ch = _value_token_channel(np.arange(P * 128))
    v[tok, ch] = v_slots
    ks = np.zeros((P // 32, 128), np.uint16)
    kz = np.zeros((P // 32, 128), np.uint16)
    ks[:, _key_meta_channel(np.arange(128))] = u16(L["k_scale"], L["k_zero"]).reshape(P // 32, 128)
    kz[:, _key_meta_channel(np.arange(128))] = u16(L["k_zero"], L["kb_scale"]).reshape(P // 32, 128)
    vs = np.zeros(P, np.uint16)
    vz = np.zeros(P, np.uint16)
    vs[_value_meta_token(np.arange(P))] = u16(L["v_scale"], L["v_zero"])
    vz[_value_meta_token(np.arange(P))] = u16(L["v_zero"], L["boost_idx"])
    return dict(kA=kA, kB=kB, v=v, ks=ks, kz=kz,
                kbs=u16(L["kb_scale"], L["v_scale"]).reshape(P // 32, k),
                vs=vs, vz=vz, idx=rec[L["boost_idx"]:L["boost_idx"] + k])


# -------------------------------------------------------------------------- pins

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


def test_storage_positions_hand_worked():
    g = _golden()
    for c, p in g["key_pos"]:
        assert oracle.key_pos(c) == p
    for KB, j, p in g["boost_pos"]:
        assert oracle.boost_pos(j, KB) == p
    for c, p in g["key_meta_pos"]:
        assert oracle.key_meta_pos(c) == p
    for t, c, word, elem in g["value_slot"]:
        assert oracle.value_slot(t, c) == 16 * word + elem
    for t, p in g["value_meta_pos"]:
        assert oracle.value_meta_pos(t) == p
    # each order is a permutation, and inverts the decoder's reading of the rule
    assert sorted(oracle.key_pos(c) for c in range(128)) == list(range(128))
    assert all(_key_channel(oracle.key_pos(c)) == c for c in range(128))
    for KB in (1, 2, 4, 8):
        assert sorted(oracle.boost_pos(j, KB) for j in range(16 * KB)) == list(range(16 * KB))
        assert all(_boost_row(oracle.boost_pos(j, KB), KB) == j for j in range(16 * KB))
    assert sorted(oracle.key_meta_pos(c) for c in range(128)) == list(range(128))
    assert all(_key_meta_channel(oracle.key_meta_pos(c)) == c for c in range(128))
    slots = [oracle.value_slot(t, c) for t in range(128) for c in range(128)]
    assert sorted(slots) == list(range(128 * 128))
    tok, ch = _value_token_channel(np.array(slots))
    assert (tok == np.repeat(np.arange(128), 128)).all() and (ch == np.tile(np.arange(128), 128)).all()
    assert sorted(oracle.value_meta_pos(t) for t in range(128)) == list(range(128))
    assert all(_value_meta_token(oracle.value_meta_pos(t)) == t for t in range(128))
    assert [oracle.elem_shift(e) for e in range(16)] == list(_shift(np.arange(16)))


@pytest.mark.parametrize("case", _golden()["words"], ids=lambda c: c["word"])
def test_key_word_packing_hand_worked(case):
    """Word 0 of token row 0 holds the key channels stored at positions 0..15; give
    element e the code case["codes"][e] through a real page and read the word back."""
    cfg = oracle.Cfg(P=32, k=0)
    K = np.zeros((cfg.P, cfg.D), np.float32)
    for e, code in enumerate(case["codes"]):
        c = int(_key_channel(e))
        K[0, c] = code
        K[1, c] = 3.0  # the group spans [0, 3]: scale 1, zero 0
    rec = oracle.quantize_page(syn.to_bits(K, F16), syn.to_bits(np.zeros_like(K), F16), cfg)
    L = oracle.layout(cfg.P, cfg.D, cfg.k, cfg.G)
    assert int(rec[L["k_codes"]:L["k_codes"] + 4].view(np.uint32)[0]) == int(case["word"], 16)


@pytest.mark.parametrize("case", _golden()["words"], ids=lambda c: c["word"])
def test_value_word_packing_hand_worked(case):
    """Word 0 of the value codes holds element e = 8a + 2(2u + v) + f <-> token 16a + 8u + f,
    channel 8v."""
    cfg = oracle.Cfg(P=32, k=0)
    V = np.zeros((cfg.P, cfg.D), np.float32)
    V[:, 1] = 3.0  # every token's range is [0, 3]: scale 1, zero 0
    for e, code in enumerate(case["codes"]):
        a, b, f = e >> 3, (e >> 1) & 3, e & 1
        V[16 * a + 8 * (b >> 1) + f, 8 * (b & 1)] = code
    rec = oracle.quantize_page(np.zeros((cfg.P, cfg.D), np.uint16), syn.to_bits(V, F16), cfg)
    L = oracle.layout(cfg.P, cfg.D, cfg.k, cfg.G)
    assert int(rec[L["v_codes"]:L["v_codes"] + 4].view(np.uint32)[0]) == int(case["word"], 16)


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


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("P,k", [(128, 0), (128, 16), (128, 32), (64, 64), (32, 128)])
def test_two_plane_split_reconstructs_4bit_codes(dtype, P, k):
    """Decoded independently: for boosted channels hi*4 + lo equals the 4-bit code of
    that channel-group, plane A scale is 4x the 4-bit scale and plane B scale the 4-bit
    scale; other channels hold their 2-bit code; values hold per-token 2-bit codes."""
    rng = np.random.default_rng(7 + k + dtype + P)
    cfg = oracle.Cfg(P=P, k=k, dtype=dtype)
    sig = np.exp(rng.standard_normal(cfg.D))
    K = syn.to_bits(rng.standard_normal((cfg.P, cfg.D)) * sig, dtype)
    V = syn.to_bits(rng.standard_normal((cfg.P, cfg.D)), dtype)
    d = _decode_record(oracle.quantize_page(K, V, cfg), P, k, dtype)
    assert d["idx"].tolist() == oracle.select_boost(K, k, dtype).tolist()
    row = {int(c): j for j, c in enumerate(d["idx"])}
    for g in range(P // 32):
        sl = slice(g * 32, (g + 1) * 32)
        for c in range(cfg.D):
            if c in row:
                j = row[c]
                c4, s4, z4 = oracle.quant_group(K[sl, c], 4, dtype)
                assert np.array_equal(d["kA"][sl, c] * 4 + d["kB"][sl, j], c4)
                assert d["kbs"][g, j] == s4
                assert oracle.value(int(d["ks"][g, c]), dtype) == 4 * oracle.value(s4, dtype)
                assert d["kz"][g, c] == z4
            else:
                c2, s2, z2 = oracle.quant_group(K[sl, c], 2, dtype)
                assert np.array_equal(d["kA"][sl, c], c2)
                assert d["ks"][g, c] == s2 and d["kz"][g, c] == z2
    for t in range(P):
        cv, sv, zv = oracle.quant_group(V[t], 2, dtype)
        assert np.array_equal(d["v"][t], cv) and d["vs"][t] == sv and d["vz"][t] == zv


def test_golden_4bit_split():
    for row in _golden()["split_4bit"]:
        assert row["hi"] * 4 + row["lo"] == row["code4"]
        assert row["code4"] >> 2 == row["hi"] and row["code4"] & 3 == row["lo"]


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_dequantize_page_matches_groupwise_dequant(dtype):
    """K^ from the two planes equals code4*s4 + mn (boosted) or code*s + mn (normal) and
    V^ equals per-token code*s + mn, exactly in fp64."""
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
    # boosting every channel (k = D) gives a much smaller key error than k = 0
    cfgD = oracle.Cfg(P=128, k=128)
    KhD, _ = oracle.dequantize_page(oracle.quantize_page(K, V, cfgD), cfgD)
    Kv = syn.from_bits(K, F16).astype(np.float64)
    assert np.abs(KhD - Kv).mean() < 0.3 * np.abs(Kh - Kv).mean()
