"""CPU oracle of the 2-bit mixed-precision KV cache — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``bit_mixed_precision_channel_b200``)
never imports it and shares no code with it: the C file ``kvq_oracle.c`` restates
every formula, the record layout and the bit packing from their definitions, and
this module restates the host-side bookkeeping (prefill split, append, flush,
attention order) the same way.

What it follows (web pages on the method, by title and section):

* "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache" (aibr.jp article),
  section 3: asymmetric quantization, Keys per channel, Values per token, a
  full-precision residual of recent tokens, streaming append.
* "Kitty: Accurate and Efficient 2-bit KV Cache Quantization with Dynamic
  Channel-wise Precision Boost" (fugumt.com summary), Abstract: rank Key channels,
  keep a small fraction at higher precision, store each mixed-precision Key page as
  two uniform 2-bit tensors in a page-centric layout.
* notes.yuuk.io wiki "KVキャッシュ量子化", open questions: magnitude-based channel
  ranking; boost ratios of 12.5% and 25%.
* "MiniKV" (f-binder summary), proposed method: prefill, then decode with 2-bit KV
  dequantized inside the attention matmul.

Readings where the pages are silent (listed again in the design notes):
scale = (max-min)/(2^b-1) in fp32, rounded up to the storage type; zero = min;
a fixed storage order of channels and tokens inside the packed rows (see
kvq_oracle.c: elem_shift, key_pos, key_meta_pos, boost_pos, value_slot,
value_meta_pos);
round half to even; clamp; scale 0 gives code 0; magnitude = max |x| over the page;
ties to the lower channel index; boost set per (page, KV head); 4-bit code =
4*hi + lo; key groups aligned to the page start; residual flushed when it holds a
whole page, before that step's attention; attention over pages in page-table order
then residual tokens, in fp64.

Parity pins: every function here is pinned by a test in ``tests/test_oracle_*.py``
against brute force, closed forms or a library routine; none is marked unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

F16 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compiles the C oracle with strict fp32 semantics (no contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i32p = ctypes.POINTER(ctypes.c_int32)
        f64p = ctypes.POINTER(ctypes.c_double)
        L.kvqo_value.restype = ctypes.c_double
        L.kvqo_value.argtypes = [ctypes.c_uint16, ctypes.c_int]
        L.kvqo_round_nearest.restype = ctypes.c_uint16
        L.kvqo_round_nearest.argtypes = [ctypes.c_double, ctypes.c_int]
        L.kvqo_round_up.restype = ctypes.c_uint16
        L.kvqo_round_up.argtypes = [ctypes.c_double, ctypes.c_int]
        L.kvqo_quant_group.restype = None
        L.kvqo_quant_group.argtypes = [u16p, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                       ctypes.c_int, u8p, u16p, u16p]
        for name in ("kvqo_elem_shift", "kvqo_key_pos", "kvqo_key_meta_pos", "kvqo_value_meta_pos"):
            getattr(L, name).restype = ctypes.c_int
            getattr(L, name).argtypes = [ctypes.c_int]
        for name in ("kvqo_boost_pos", "kvqo_value_slot"):
            getattr(L, name).restype = ctypes.c_int
            getattr(L, name).argtypes = [ctypes.c_int, ctypes.c_int]
        L.kvqo_layout.restype = None
        L.kvqo_layout.argtypes = [ctypes.c_int] * 4 + [ctypes.POINTER(ctypes.c_long)]
        L.kvqo_select_boost.restype = None
        L.kvqo_select_boost.argtypes = [u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, u8p]
        L.kvqo_quantize_page.restype = None
        L.kvqo_quantize_page.argtypes = [u16p, u16p, ctypes.c_long] + [ctypes.c_int] * 5 + [u8p]
        f32p = ctypes.POINTER(ctypes.c_float)
        L.kvqo_quantize_page_ex.restype = None
        L.kvqo_quantize_page_ex.argtypes = [u16p, u16p, ctypes.c_long] + [ctypes.c_int] * 5 + [
            f32p, ctypes.c_int, u8p]
        L.kvqo_prefill_attention.restype = None
        L.kvqo_prefill_attention.argtypes = [u16p, u16p, u16p] + [ctypes.c_int] * 5 + [ctypes.c_double, f64p, f64p]
        L.kvqo_retain.restype = ctypes.c_int
        L.kvqo_retain.argtypes = [f64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p]
        L.kvqo_select_boost_query.restype = None
        L.kvqo_select_boost_query.argtypes = [u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              f32p, ctypes.c_int, u8p]
        L.kvqo_dequantize_page.restype = None
        L.kvqo_dequantize_page.argtypes = [u8p] + [ctypes.c_int] * 5 + [f64p, f64p]
        L.kvqo_decode_unit.restype = None
        L.kvqo_decode_unit.argtypes = [u8p, ctypes.c_int, ctypes.c_int, i32p, ctypes.c_int,
                                       u16p, u16p, ctypes.c_int, u16p] + [ctypes.c_int] * 6 + [
                                           ctypes.c_double, f64p]
        _lib = L
    return _lib


def _p(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ------------------------------------------------------------------ scalar helpers

def value(bits: int, dtype: int) -> float:
    """Exact value of a 16-bit pattern of the storage type."""
    return lib().kvqo_value(int(bits), dtype)


def values(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact fp64 values of an array of 16-bit patterns (vectorised restatement)."""
    b = np.asarray(bits, dtype=np.uint16)
    if dtype == BF16:
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return b.view(np.float16).astype(np.float64)


def round_up(x: float, dtype: int) -> int:
    return int(lib().kvqo_round_up(float(x), dtype))


def round_nearest(x: float, dtype: int) -> int:
    return int(lib().kvqo_round_nearest(float(x), dtype))


# ------------------------------------------------------------------------ quantizer

def quant_group(x_bits: np.ndarray, bits: int, dtype: int):
    """Asymmetric min/max quantization of one group -> (codes, scale_bits, zero_bits)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n = x.size
    codes = np.zeros(n, np.uint8)
    sb = ctypes.c_uint16()
    zb = ctypes.c_uint16()
    lib().kvqo_quant_group(_p(x, ctypes.c_uint16), n, 1, bits, dtype, _p(codes, ctypes.c_uint8),
                           ctypes.byref(sb), ctypes.byref(zb))
    return codes, int(sb.value), int(zb.value)


# ---------------------------------------------------------------------- page layout

def elem_shift(e: int) -> int:
    """Bit position of element e (0..15) of a 32-bit code word."""
    return lib().kvqo_elem_shift(e)


def key_pos(c: int) -> int:
    """Storage position of key channel c in plane-A code rows."""
    return lib().kvqo_key_pos(c)


def key_meta_pos(c: int) -> int:
    """Storage position of key channel c in the plane-A scale and zero rows."""
    return lib().kvqo_key_meta_pos(c)


def boost_pos(j: int, KB: int) -> int:
    """Storage position of boosted row j in plane-B rows (KB = boosted channels / 16)."""
    return lib().kvqo_boost_pos(j, KB)


def value_slot(t: int, c: int) -> int:
    """Slot (16 * word + element) of the value code of token t, channel c."""
    return lib().kvqo_value_slot(t, c)


def value_meta_pos(t: int) -> int:
    """Storage position of token t in the value scale and zero rows."""
    return lib().kvqo_value_meta_pos(t)


LAYOUT_KEYS = ("k_codes", "kb_codes", "v_codes", "k_scale", "k_zero", "kb_scale",
               "v_scale", "v_zero", "boost_idx", "payload_bytes", "record_bytes")


def layout(P: int, D: int, k: int, G: int) -> dict:
    out = (ctypes.c_long * 11)()
    lib().kvqo_layout(P, D, k, G, out)
    return dict(zip(LAYOUT_KEYS, [int(v) for v in out]))


@dataclass(frozen=True)
class Cfg:
    """Shape of one layer's cache (oracle's own copy of the configuration)."""
    D: int = 128
    Hq: int = 1
    Hkv: int = 1
    P: int = 128
    G: int = 32
    k: int = 16
    dtype: int = F16

    @property
    def gqa(self) -> int:
        return self.Hq // self.Hkv

    @property
    def record_bytes(self) -> int:
        return layout(self.P, self.D, self.k, self.G)["record_bytes"]


def select_boost(K_bits: np.ndarray, k: int, dtype: int) -> np.ndarray:
    """Boosted channels of one page: K_bits [P][D] -> ascending uint8[k]."""
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    P, D = K.shape
    idx = np.zeros(k, np.uint8)
    lib().kvqo_select_boost(_p(K, ctypes.c_uint16), D, P, D, k, dtype, _p(idx, ctypes.c_uint8))
    return idx


def select_boost_query(K_bits: np.ndarray, n: int, weight: np.ndarray, dtype: int) -> np.ndarray:
    """Query-aware boosted channels of one page (MixKVQ reading): K_bits [P][D], weight
    float32[D] -> ascending uint8[n]."""
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    w = np.ascontiguousarray(weight, dtype=np.float32)
    P, D = K.shape
    idx = np.zeros(n, np.uint8)
    lib().kvqo_select_boost_query(_p(K, ctypes.c_uint16), D, P, D, n, _p(w, ctypes.c_float), dtype,
                                  _p(idx, ctypes.c_uint8))
    return idx


def quantize_page_ex(K_bits: np.ndarray, V_bits: np.ndarray, cfg: Cfg, n_boost: int | None = None,
                     weight: np.ndarray | None = None) -> np.ndarray:
    """quantize_page with n_boost <= cfg.k boosted channels (the per-head boost count)
    and, when weight is given, the query-aware ranking."""
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    assert K.shape == (cfg.P, cfg.D) and V.shape == (cfg.P, cfg.D)
    n = cfg.k if n_boost is None else int(n_boost)
    assert 0 <= n <= cfg.k
    w = None if weight is None else np.ascontiguousarray(weight, dtype=np.float32)
    rec = np.zeros(cfg.record_bytes, np.uint8)
    lib().kvqo_quantize_page_ex(_p(K, ctypes.c_uint16), _p(V, ctypes.c_uint16), cfg.D, cfg.P, cfg.D, cfg.G,
                                cfg.k, n, None if w is None else _p(w, ctypes.c_float), cfg.dtype,
                                _p(rec, ctypes.c_uint8))
    return rec


def prefill_attention(Q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray, dtype: int,
                      sm_scale: float):
    """Causal prefill attention and cumulative attention scores (MiniKV reading):
    Q [L][Hq][D], K and V [L][Hkv][D] patterns -> (O fp64 [L][Hq][D], A fp64 [Hkv][L])."""
    Q = np.ascontiguousarray(Q_bits, dtype=np.uint16)
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    L, Hq, D = Q.shape
    Hkv = K.shape[1]
    O = np.zeros((L, Hq, D), np.float64)
    A = np.zeros((Hkv, L), np.float64)
    lib().kvqo_prefill_attention(_p(Q, ctypes.c_uint16), _p(K, ctypes.c_uint16), _p(V, ctypes.c_uint16), L, Hq,
                                 Hkv, D, dtype, float(sm_scale), _p(O, ctypes.c_double), _p(A, ctypes.c_double))
    return O, A


def retain(A_row: np.ndarray, n_heavy: int, n_recent: int) -> np.ndarray:
    """Kept positions of one KV head: the last n_recent, plus the n_heavy best-scored
    of the others (ties to the lower position), ascending."""
    a = np.ascontiguousarray(A_row, dtype=np.float64)
    keep = np.zeros(max(1, a.size), np.int32)
    n = lib().kvqo_retain(_p(a, ctypes.c_double), a.size, n_heavy, n_recent, _p(keep, ctypes.c_int32))
    return keep[:n]


def quantize_page(K_bits: np.ndarray, V_bits: np.ndarray, cfg: Cfg) -> np.ndarray:
    """One page of one KV head ([P][D] each) -> record bytes (uint8[record_bytes])."""
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    assert K.shape == (cfg.P, cfg.D) and V.shape == (cfg.P, cfg.D)
    rec = np.zeros(cfg.record_bytes, np.uint8)
    lib().kvqo_quantize_page(_p(K, ctypes.c_uint16), _p(V, ctypes.c_uint16), cfg.D, cfg.P, cfg.D,
                             cfg.G, cfg.k, cfg.dtype, _p(rec, ctypes.c_uint8))
    return rec


def dequantize_page(rec: np.ndarray, cfg: Cfg):
    """Record -> (K^, V^) as fp64 [P][D] each."""
    r = np.ascontiguousarray(rec, dtype=np.uint8)
    Kh = np.zeros((cfg.P, cfg.D), np.float64)
    Vh = np.zeros((cfg.P, cfg.D), np.float64)
    lib().kvqo_dequantize_page(_p(r, ctypes.c_uint8), cfg.P, cfg.D, cfg.G, cfg.k, cfg.dtype,
                               _p(Kh, ctypes.c_double), _p(Vh, ctypes.c_double))
    return Kh, Vh


def decode_unit(pool: np.ndarray, cfg: Cfg, head: int, pages, res_k: np.ndarray,
                res_v: np.ndarray, q: np.ndarray, sm_scale: float) -> np.ndarray:
    """Attention of the gqa query heads of one KV head of one sequence (fp64).

    pool: uint8 [pool_pages][Hkv][record_bytes]; pages: the sequence's page ids in
    token order; res_k/res_v: [res_len][D] 16-bit patterns; q: [gqa][D] patterns.
    Returns [gqa][D] fp64."""
    pool = np.ascontiguousarray(pool, dtype=np.uint8)
    pg = np.ascontiguousarray(np.asarray(pages, dtype=np.int32))
    rk = np.ascontiguousarray(res_k, dtype=np.uint16).reshape(-1, cfg.D)
    rv = np.ascontiguousarray(res_v, dtype=np.uint16).reshape(-1, cfg.D)
    qq = np.ascontiguousarray(q, dtype=np.uint16).reshape(cfg.gqa, cfg.D)
    out = np.zeros((cfg.gqa, cfg.D), np.float64)
    if rk.shape[0] == 0:
        rk = np.zeros((1, cfg.D), np.uint16)
        rv = np.zeros((1, cfg.D), np.uint16)
        n_res = 0
    else:
        n_res = rk.shape[0]
    lib().kvqo_decode_unit(_p(pool, ctypes.c_uint8), cfg.Hkv, head, _p(pg, ctypes.c_int32),
                           pg.size, _p(rk, ctypes.c_uint16), _p(rv, ctypes.c_uint16), n_res,
                           _p(qq, ctypes.c_uint16), cfg.gqa, cfg.P, cfg.D, cfg.G, cfg.k,
                           cfg.dtype, float(sm_scale), _p(out, ctypes.c_double))
    return out


# ------------------------------------------------------------ host-side pipeline

@dataclass
class Sequence:
    pages: list = field(default_factory=list)
    res_k: list = field(default_factory=list)  # per kv head: list of [D] uint16 rows
    res_v: list = field(default_factory=list)


class OracleCache:
    """The decode pipeline of one layer, restated on the host.

    prefill: a prompt of L tokens becomes floor(L/P) pages (quantized in order into
    the pages the caller names) and L mod P residual tokens.
    append: one token per sequence goes to the end of its residual window.
    flush: a window holding P tokens becomes one page (into the page the caller
    names) and empties.  A decode step is append, then flush, then attention.
    attend: per query head, softmax attention over the pages then the residual."""

    def __init__(self, cfg: Cfg, batch: int, pool_pages: int):
        self.cfg = cfg
        self.pool = np.zeros((pool_pages, cfg.Hkv, cfg.record_bytes), np.uint8)
        self.seqs = [Sequence(res_k=[[] for _ in range(cfg.Hkv)],
                              res_v=[[] for _ in range(cfg.Hkv)]) for _ in range(batch)]

    def write_page(self, page: int, K_page: np.ndarray, V_page: np.ndarray):
        """K_page, V_page: [P][Hkv][D] token-major patterns."""
        for h in range(self.cfg.Hkv):
            self.pool[page, h] = quantize_page(K_page[:, h, :], V_page[:, h, :], self.cfg)

    def prefill(self, b: int, K: np.ndarray, V: np.ndarray, pages):
        """K, V: [L][Hkv][D] patterns; pages: floor(L/P) page ids."""
        P = self.cfg.P
        n_full = K.shape[0] // P
        assert len(pages) == n_full
        for i in range(n_full):
            self.write_page(int(pages[i]), K[i * P:(i + 1) * P], V[i * P:(i + 1) * P])
            self.seqs[b].pages.append(int(pages[i]))
        for h in range(self.cfg.Hkv):
            self.seqs[b].res_k[h] = [K[t, h].copy() for t in range(n_full * P, K.shape[0])]
            self.seqs[b].res_v[h] = [V[t, h].copy() for t in range(n_full * P, V.shape[0])]

    def res_len(self, b: int) -> int:
        return len(self.seqs[b].res_k[0])

    def append(self, k_new: np.ndarray, v_new: np.ndarray):
        """k_new, v_new: [B][Hkv][D] patterns."""
        for b, s in enumerate(self.seqs):
            assert self.res_len(b) < self.cfg.P, "append into a full residual window"
            for h in range(self.cfg.Hkv):
                s.res_k[h].append(k_new[b, h].copy())
                s.res_v[h].append(v_new[b, h].copy())

    def flush(self, new_page):
        """new_page[b]: page id for b if its window is full.  Returns flushed b's."""
        flushed = []
        for b, s in enumerate(self.seqs):
            if self.res_len(b) == self.cfg.P:
                page = int(new_page[b])
                Kp = np.stack([np.stack(s.res_k[h]) for h in range(self.cfg.Hkv)], axis=1)
                Vp = np.stack([np.stack(s.res_v[h]) for h in range(self.cfg.Hkv)], axis=1)
                self.write_page(page, Kp, Vp)
                s.pages.append(page)
                for h in range(self.cfg.Hkv):
                    s.res_k[h] = []
                    s.res_v[h] = []
                flushed.append(b)
        return flushed

    def attend_unit(self, b: int, kvh: int, q: np.ndarray, sm_scale: float) -> np.ndarray:
        """q: [Hq][D] patterns of sequence b -> out [gqa][D] of KV head kvh (fp64)."""
        g = self.cfg.gqa
        s = self.seqs[b]
        rk = np.stack(s.res_k[kvh]) if s.res_k[kvh] else np.zeros((0, self.cfg.D), np.uint16)
        rv = np.stack(s.res_v[kvh]) if s.res_v[kvh] else np.zeros((0, self.cfg.D), np.uint16)
        return decode_unit(self.pool, self.cfg, kvh, s.pages, rk, rv, q[kvh * g:(kvh + 1) * g],
                           sm_scale)

    def attend(self, q: np.ndarray, sm_scale: float) -> np.ndarray:
        """q: [B][Hq][D] patterns -> out [B][Hq][D] fp64."""
        B = len(self.seqs)
        out = np.zeros((B, self.cfg.Hq, self.cfg.D), np.float64)
        g = self.cfg.gqa
        for b in range(B):
            for h in range(self.cfg.Hkv):
                out[b, h * g:(h + 1) * g] = self.attend_unit(b, h, q[b], sm_scale)
        return out
