"""ctypes binding of libkvq.so — argument marshalling only.

Every function has the name of the C entry point it calls (without the ``kvq_``
prefix) and passes device pointers (``tensor.data_ptr()``), sizes and the current
PyTorch CUDA stream straight through.  All computation happens in the library's
CUDA kernels; there is no fallback of any kind: if the library is missing, was not
built, or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

__all__ = [
    "KVQError", "Config", "Source", "library_path", "load", "status_string", "check_config",
    "page_layout", "page_bytes", "select_boost_channels", "quantize_page_keys",
    "quantize_values", "quantize_pages", "append_token", "flush_residual",
    "decode_workspace_bytes", "decode_attention", "decode_attention_static", "STATIC_SCRATCH_BYTES",
    "quantize_pages_ex", "dense_page_bytes", "decode_attention_dense",
    "prefill_workspace_bytes", "prefill_attention", "retain_tokens", "gather_tokens",
    "F16", "BF16", "torch_dtype",
    "DEV_ERR_PAGE_RANGE", "DEV_ERR_RESIDUAL", "DEV_ERR_TABLE_FULL", "DEV_ERR_TIMEOUT",
    "DEV_ERR_LENGTH", "DEV_ERR_RANGE",
]

F16 = 0
BF16 = 1
DEV_ERR_PAGE_RANGE = 1
DEV_ERR_RESIDUAL = 2
DEV_ERR_TABLE_FULL = 4
DEV_ERR_TIMEOUT = 8
DEV_ERR_LENGTH = 16
DEV_ERR_RANGE = 32
STATIC_SCRATCH_BYTES = 16 << 20  # KVQ_STATIC_SCRATCH_BYTES

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libkvq.so")


class KVQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "head_dim", "num_q_heads", "num_kv_heads", "page_tokens", "key_group", "key_bits",
        "boost_bits", "value_bits", "num_boost", "dtype")]


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "k_codes", "kb_codes", "v_codes", "k_scale", "k_zero", "kb_scale", "v_scale", "v_zero",
        "boost_idx", "payload_bytes", "record_bytes")]


class _BoostOptions(ctypes.Structure):
    _fields_ = [("query_weight", ctypes.c_void_p), ("boost_per_head", ctypes.c_void_p)]


class _Source(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("page_stride", ctypes.c_int64),
                ("token_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64)]


@dataclass(frozen=True)
class Config:
    """Cache shape of one attention layer (mirrors kvq_config)."""
    head_dim: int = 128
    num_q_heads: int = 32
    num_kv_heads: int = 8
    page_tokens: int = 128
    key_group: int = 32
    num_boost: int = 32
    dtype: int = F16
    key_bits: int = 2
    boost_bits: int = 4
    value_bits: int = 2

    @property
    def gqa(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def c(self) -> _Config:
        return _Config(self.head_dim, self.num_q_heads, self.num_kv_heads, self.page_tokens,
                       self.key_group, self.key_bits, self.boost_bits, self.value_bits,
                       self.num_boost, self.dtype)


def torch_dtype(dtype: int) -> torch.dtype:
    return torch.bfloat16 if dtype == BF16 else torch.float16


@dataclass
class Source:
    """Pages of a 16-bit tensor: element (page i, token t, kv head h, channel c) is at
    tensor.flatten()[i*page_stride + t*token_stride + h*head_stride + c]."""
    tensor: torch.Tensor
    page_stride: int
    token_stride: int
    head_stride: int

    @staticmethod
    def token_major(x: torch.Tensor, cfg: Config, first_token: int = 0) -> "Source":
        """x: [tokens][Hkv][D] contiguous; pages start at token `first_token`."""
        assert x.is_contiguous() and x.dim() == 3
        H, D, P = cfg.num_kv_heads, cfg.head_dim, cfg.page_tokens
        return Source(x[first_token:] if first_token else x, P * H * D, H * D, D)

    def c(self) -> _Source:
        return _Source(self.tensor.data_ptr(), self.page_stride, self.token_stride, self.head_stride)


_lib = None


def load():
    """Loads libkvq.so once; raises if it is missing."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"libkvq.so not found at {path}; build it with "
                               "`python -m bit_mixed_precision_channel_b200.build`")
        L = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        cfgp = ctypes.POINTER(_Config)
        L.kvq_status_string.restype = ctypes.c_char_p
        L.kvq_status_string.argtypes = [ctypes.c_int]
        L.kvq_check_config.restype = ctypes.c_int
        L.kvq_check_config.argtypes = [cfgp]
        L.kvq_page_layout.restype = ctypes.c_int
        L.kvq_page_layout.argtypes = [cfgp, ctypes.POINTER(_Layout)]
        L.kvq_page_bytes.restype = sz
        L.kvq_page_bytes.argtypes = [cfgp]
        for name in ("kvq_select_boost_channels", "kvq_quantize_page_keys", "kvq_quantize_values"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = [cfgp, _Source, vp, i32, vp, i64, vp, vp]
        L.kvq_quantize_pages.restype = ctypes.c_int
        L.kvq_quantize_pages.argtypes = [cfgp, _Source, _Source, vp, i32, vp, i64, vp, vp]
        L.kvq_append_token.restype = ctypes.c_int
        L.kvq_append_token.argtypes = [cfgp, i32, vp, vp, vp, vp, vp, vp, vp]
        L.kvq_flush_residual.restype = ctypes.c_int
        L.kvq_flush_residual.argtypes = [cfgp, i32, vp, vp, vp, vp, vp, i32, vp, vp, i64, vp, vp]
        L.kvq_append_flush.restype = ctypes.c_int
        L.kvq_append_flush.argtypes = [cfgp, i32, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i64,
                                       ctypes.POINTER(_BoostOptions), vp, vp, vp]
        L.kvq_dense_page_bytes.restype = sz
        L.kvq_dense_page_bytes.argtypes = [cfgp]
        L.kvq_decode_attention_dense.restype = ctypes.c_int
        L.kvq_decode_attention_dense.argtypes = [cfgp, vp, i64, vp, i32, vp, i32, vp, ctypes.c_float, vp, vp, sz,
                                                 vp, vp]
        L.kvq_prefill_workspace_bytes.restype = sz
        L.kvq_prefill_workspace_bytes.argtypes = [cfgp, i32]
        L.kvq_prefill_attention.restype = ctypes.c_int
        L.kvq_prefill_attention.argtypes = [cfgp, vp, vp, vp, i32, ctypes.c_float, vp, vp, vp, sz, vp]
        L.kvq_retain_tokens.restype = ctypes.c_int
        L.kvq_retain_tokens.argtypes = [cfgp, vp, i32, i32, i32, vp, vp, vp]
        L.kvq_gather_tokens.restype = ctypes.c_int
        L.kvq_gather_tokens.argtypes = [cfgp, vp, vp, i32, vp, i32, vp, vp, vp, vp]
        optp = ctypes.POINTER(_BoostOptions)
        L.kvq_quantize_pages_ex.restype = ctypes.c_int
        L.kvq_quantize_pages_ex.argtypes = [cfgp, _Source, _Source, vp, i32, vp, i64, optp, vp, vp]
        L.kvq_flush_residual_ex.restype = ctypes.c_int
        L.kvq_flush_residual_ex.argtypes = [cfgp, i32, vp, vp, vp, vp, vp, i32, vp, vp, i64, optp, vp, vp]
        L.kvq_decode_workspace_bytes.restype = sz
        L.kvq_decode_workspace_bytes.argtypes = [cfgp, i32, i32]
        L.kvq_decode_attention.restype = ctypes.c_int
        L.kvq_decode_attention.argtypes = [cfgp, vp, i64, vp, i32, vp, i32, vp, vp, vp, vp,
                                           ctypes.c_float, vp, vp, sz, vp, vp]
        L.kvq_decode_attention_static.restype = ctypes.c_int
        L.kvq_decode_attention_static.argtypes = [cfgp, vp, i64, vp, i32, vp, i32, vp, vp, vp, vp,
                                                  ctypes.c_float, vp, vp, vp]
        _lib = L
    return _lib


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _check(fn: str, status: int):
    if status != 0:
        raise KVQError(fn, status)


def _cuda(*tensors, stream=None):
    """Every tensor must be device memory of one device, the current one: the library
    launches on the current device and its stream, and a pointer into another GPU's
    memory would fault there instead of failing cleanly."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("kvq calls take CUDA tensors (device memory)")
        if dev is None:
            dev = t.device.index
        elif t.device.index != dev:
            raise ValueError(f"kvq calls take tensors of one device: cuda:{dev} and cuda:{t.device.index}")
    if dev is None:
        return
    cur = torch.cuda.current_device()
    if dev != cur:
        raise ValueError(f"tensors are on cuda:{dev} but the current device is cuda:{cur}; "
                         f"make the call under torch.cuda.device({dev})")
    if stream is not None and getattr(stream, "device", None) is not None and stream.device.index != dev:
        raise ValueError(f"stream of cuda:{stream.device.index} for tensors on cuda:{dev}")


def _need(name: str, t, dtype=None, numel: int | None = None, dim: int | None = None):
    """The library takes plain pointers: a tensor must be dense, of the element type the
    call reads, and at least as large as the call's extent."""
    if t is None:
        return
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, the call reads {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, not {t.dim()}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the call reads {numel}")


def _need_source(name: str, src, cfg: Config, n_pages: int):
    if src is None:
        return
    extent = 0
    if n_pages > 0:
        extent = ((n_pages - 1) * src.page_stride + (cfg.page_tokens - 1) * src.token_stride +
                  (cfg.num_kv_heads - 1) * src.head_stride + cfg.head_dim)
    _need(name, src.tensor, torch_dtype(cfg.dtype), extent)


def status_string(status: int) -> str:
    return load().kvq_status_string(status).decode()


def check_config(cfg: Config) -> int:
    return load().kvq_check_config(ctypes.byref(cfg.c()))


def page_layout(cfg: Config) -> dict:
    out = _Layout()
    _check("kvq_page_layout", load().kvq_page_layout(ctypes.byref(cfg.c()), ctypes.byref(out)))
    return {n: int(getattr(out, n)) for n, _ in _Layout._fields_}


def page_bytes(cfg: Config) -> int:
    return int(load().kvq_page_bytes(ctypes.byref(cfg.c())))


def _boost_options(cfg: Config, query_weight, boost_per_head):
    """Checks and marshals the boost options (device float32 [Hkv][D] weights, device
    int32 [Hkv] counts); None for both gives a null pointer (the plain behaviour)."""
    _need("query_weight", query_weight, torch.float32, cfg.num_kv_heads * cfg.head_dim)
    _need("boost_per_head", boost_per_head, torch.int32, cfg.num_kv_heads)
    if query_weight is None and boost_per_head is None:
        return None
    return ctypes.byref(_BoostOptions(_ptr(query_weight), _ptr(boost_per_head)))


def _quant(fn, cfg, src_k, src_v, dst_pages, pool, err, stream, query_weight=None, boost_per_head=None):
    _need("dst_pages", dst_pages, torch.int32)
    _need("pool", pool, torch.uint8)
    _need("err", err, torch.int32, 1)
    _need_source("k source", src_k, cfg, dst_pages.numel())
    _need_source("v source", src_v, cfg, dst_pages.numel())
    _cuda(dst_pages, pool, err, src_k.tensor if src_k is not None else None,
          src_v.tensor if src_v is not None else None, stream=stream)
    pool_pages = pool.numel() // (cfg.num_kv_heads * page_bytes(cfg))
    L = load()
    n = dst_pages.numel()
    if fn == "kvq_quantize_pages_ex":
        _cuda(query_weight, boost_per_head, pool, stream=stream)
        st = L.kvq_quantize_pages_ex(ctypes.byref(cfg.c()), src_k.c(), src_v.c(), dst_pages.data_ptr(), n,
                                     pool.data_ptr(), pool_pages, _boost_options(cfg, query_weight, boost_per_head),
                                     _ptr(err), _stream(stream))
    elif fn == "kvq_quantize_pages":
        st = L.kvq_quantize_pages(ctypes.byref(cfg.c()), src_k.c(), src_v.c(), dst_pages.data_ptr(), n,
                                  pool.data_ptr(), pool_pages, _ptr(err), _stream(stream))
    else:
        src = src_k if src_k is not None else src_v
        st = getattr(L, fn)(ctypes.byref(cfg.c()), src.c(), dst_pages.data_ptr(), n, pool.data_ptr(),
                            pool_pages, _ptr(err), _stream(stream))
    _check(fn, st)


def select_boost_channels(cfg: Config, k: Source, dst_pages: torch.Tensor, pool: torch.Tensor,
                          err: torch.Tensor | None = None, stream=None):
    _quant("kvq_select_boost_channels", cfg, k, None, dst_pages, pool, err, stream)


def quantize_page_keys(cfg: Config, k: Source, dst_pages: torch.Tensor, pool: torch.Tensor,
                       err: torch.Tensor | None = None, stream=None):
    _quant("kvq_quantize_page_keys", cfg, k, None, dst_pages, pool, err, stream)


def quantize_values(cfg: Config, v: Source, dst_pages: torch.Tensor, pool: torch.Tensor,
                    err: torch.Tensor | None = None, stream=None):
    _quant("kvq_quantize_values", cfg, None, v, dst_pages, pool, err, stream)


def quantize_pages(cfg: Config, k: Source, v: Source, dst_pages: torch.Tensor, pool: torch.Tensor,
                   err: torch.Tensor | None = None, stream=None):
    _quant("kvq_quantize_pages", cfg, k, v, dst_pages, pool, err, stream)


def quantize_pages_ex(cfg: Config, k: Source, v: Source, dst_pages: torch.Tensor, pool: torch.Tensor,
                      err: torch.Tensor | None = None, stream=None, query_weight=None, boost_per_head=None):
    """quantize_pages with the boost options: query_weight (float32 [Hkv][D], the
    query-aware ranking) and boost_per_head (int32 [Hkv], boosted channels per head)."""
    _quant("kvq_quantize_pages_ex", cfg, k, v, dst_pages, pool, err, stream, query_weight, boost_per_head)


def append_token(cfg: Config, k_new, v_new, res_k, res_v, res_len, err=None, stream=None):
    batch = res_len.numel()
    dt, H, P, D = torch_dtype(cfg.dtype), cfg.num_kv_heads, cfg.page_tokens, cfg.head_dim
    _need("res_len", res_len, torch.int32)
    _need("k_new", k_new, dt, batch * H * D)
    _need("v_new", v_new, dt, batch * H * D)
    _need("res_k", res_k, dt, batch * H * P * D)
    _need("res_v", res_v, dt, batch * H * P * D)
    _need("err", err, torch.int32, 1)
    _cuda(k_new, v_new, res_k, res_v, res_len, err, stream=stream)
    _check("kvq_append_token", load().kvq_append_token(
        ctypes.byref(cfg.c()), batch, k_new.data_ptr(), v_new.data_ptr(), res_k.data_ptr(),
        res_v.data_ptr(), res_len.data_ptr(), _ptr(err), _stream(stream)))


def flush_residual(cfg: Config, res_k, res_v, res_len, new_page, page_table, num_pages, pool,
                   err=None, stream=None, query_weight=None, boost_per_head=None):
    _need("page_table", page_table, torch.int32, dim=2)
    batch, max_pages = page_table.shape
    dt, H, P, D = torch_dtype(cfg.dtype), cfg.num_kv_heads, cfg.page_tokens, cfg.head_dim
    _need("res_k", res_k, dt, batch * H * P * D)
    _need("res_v", res_v, dt, batch * H * P * D)
    for name, t in (("res_len", res_len), ("new_page", new_page), ("num_pages", num_pages)):
        _need(name, t, torch.int32, batch)
    _need("pool", pool, torch.uint8)
    _need("err", err, torch.int32, 1)
    _cuda(res_k, res_v, res_len, new_page, page_table, num_pages, pool, err, query_weight, boost_per_head,
          stream=stream)
    pool_pages = pool.numel() // (cfg.num_kv_heads * page_bytes(cfg))
    opts = _boost_options(cfg, query_weight, boost_per_head)
    if opts is None:
        _check("kvq_flush_residual", load().kvq_flush_residual(
            ctypes.byref(cfg.c()), batch, res_k.data_ptr(), res_v.data_ptr(), res_len.data_ptr(),
            new_page.data_ptr(), page_table.data_ptr(), max_pages, num_pages.data_ptr(), pool.data_ptr(),
            pool_pages, _ptr(err), _stream(stream)))
    else:
        _check("kvq_flush_residual_ex", load().kvq_flush_residual_ex(
            ctypes.byref(cfg.c()), batch, res_k.data_ptr(), res_v.data_ptr(), res_len.data_ptr(),
            new_page.data_ptr(), page_table.data_ptr(), max_pages, num_pages.data_ptr(), pool.data_ptr(),
            pool_pages, opts, _ptr(err), _stream(stream)))


def append_flush(cfg: Config, k_new, v_new, res_k, res_v, res_len, new_page, page_table, num_pages, pool,
                 counters, err=None, stream=None, query_weight=None, boost_per_head=None):
    """append_token followed by flush_residual, in one launch (kvq_append_flush).
    counters: int32[batch], zero before the first call; every call leaves it zero."""
    _need("page_table", page_table, torch.int32, dim=2)
    batch, max_pages = page_table.shape
    dt, H, P, D = torch_dtype(cfg.dtype), cfg.num_kv_heads, cfg.page_tokens, cfg.head_dim
    _need("k_new", k_new, dt, batch * H * D)
    _need("v_new", v_new, dt, batch * H * D)
    _need("res_k", res_k, dt, batch * H * P * D)
    _need("res_v", res_v, dt, batch * H * P * D)
    for name, t in (("res_len", res_len), ("new_page", new_page), ("num_pages", num_pages),
                    ("counters", counters)):
        _need(name, t, torch.int32, batch)
    _need("pool", pool, torch.uint8)
    _need("err", err, torch.int32, 1)
    _cuda(k_new, v_new, res_k, res_v, res_len, new_page, page_table, num_pages, pool, counters, err,
          query_weight, boost_per_head, stream=stream)
    pool_pages = pool.numel() // (cfg.num_kv_heads * page_bytes(cfg))
    opts = _boost_options(cfg, query_weight, boost_per_head)
    _check("kvq_append_flush", load().kvq_append_flush(
        ctypes.byref(cfg.c()), batch, k_new.data_ptr(), v_new.data_ptr(), res_k.data_ptr(), res_v.data_ptr(),
        res_len.data_ptr(), new_page.data_ptr(), page_table.data_ptr(), max_pages, num_pages.data_ptr(),
        pool.data_ptr(), pool_pages, opts, counters.data_ptr(), _ptr(err), _stream(stream)))


def decode_workspace_bytes(cfg: Config, batch: int, max_pages: int) -> int:
    return int(load().kvq_decode_workspace_bytes(ctypes.byref(cfg.c()), batch, max_pages))


def _need_decode(cfg: Config, pool, q, page_table, num_pages, res_k, res_v, res_len, out, err):
    _need("page_table", page_table, torch.int32, dim=2)
    batch = page_table.shape[0]
    dt, H, P, D = torch_dtype(cfg.dtype), cfg.num_kv_heads, cfg.page_tokens, cfg.head_dim
    _need("pool", pool, torch.uint8)
    _need("q", q, dt, batch * cfg.num_q_heads * D)
    _need("out", out, torch.float32, batch * cfg.num_q_heads * D)
    _need("num_pages", num_pages, torch.int32, batch)
    _need("res_len", res_len, torch.int32, batch)
    _need("res_k", res_k, dt, batch * H * P * D)
    _need("res_v", res_v, dt, batch * H * P * D)
    _need("err", err, torch.int32, 1)


def decode_attention(cfg: Config, pool, q, page_table, num_pages, res_k, res_v, res_len, out,
                     workspace, sm_scale: float | None = None, err=None, stream=None):
    _need_decode(cfg, pool, q, page_table, num_pages, res_k, res_v, res_len, out, err)
    _need("workspace", workspace, torch.uint8)
    _cuda(pool, q, page_table, num_pages, res_k, res_v, res_len, out, workspace, err, stream=stream)
    batch, max_pages = page_table.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    pool_pages = pool.numel() // (cfg.num_kv_heads * page_bytes(cfg))
    _check("kvq_decode_attention", load().kvq_decode_attention(
        ctypes.byref(cfg.c()), pool.data_ptr(), pool_pages, q.data_ptr(), batch, page_table.data_ptr(),
        max_pages, num_pages.data_ptr(), res_k.data_ptr(), res_v.data_ptr(), res_len.data_ptr(),
        float(sm_scale), out.data_ptr(), workspace.data_ptr(), workspace.numel(), _ptr(err),
        _stream(stream)))


def decode_attention_static(cfg: Config, pool, q, page_table, num_pages, res_k, res_v, res_len, out,
                            sm_scale: float | None = None, err=None, stream=None):
    """decode_attention for callers that cannot allocate device memory: the split-K
    scratch is the library's own static 16 MiB device buffer (no workspace argument).
    Calls on one device share that buffer, so they must not overlap on the GPU; the
    first call on a device must not be made during stream capture."""
    _need_decode(cfg, pool, q, page_table, num_pages, res_k, res_v, res_len, out, err)
    _cuda(pool, q, page_table, num_pages, res_k, res_v, res_len, out, err, stream=stream)
    batch, max_pages = page_table.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    pool_pages = pool.numel() // (cfg.num_kv_heads * page_bytes(cfg))
    _check("kvq_decode_attention_static", load().kvq_decode_attention_static(
        ctypes.byref(cfg.c()), pool.data_ptr(), pool_pages, q.data_ptr(), batch, page_table.data_ptr(),
        max_pages, num_pages.data_ptr(), res_k.data_ptr(), res_v.data_ptr(), res_len.data_ptr(),
        float(sm_scale), out.data_ptr(), _ptr(err), _stream(stream)))


def dense_page_bytes(cfg: Config) -> int:
    return int(load().kvq_dense_page_bytes(ctypes.byref(cfg.c())))


def decode_attention_dense(cfg: Config, pool, q, page_table, seq_len, out, workspace,
                           sm_scale: float | None = None, err=None, stream=None):
    """Decode attention over an unquantized paged cache (the full-precision baseline):
    pool dtype [pool_pages][Hkv][2][P][D], page_table int32 [B][max_pages], seq_len int32 [B]."""
    dt = torch_dtype(cfg.dtype)
    _need("page_table", page_table, torch.int32, dim=2)
    batch, max_pages = page_table.shape
    _need("pool", pool, dt)
    _need("seq_len", seq_len, torch.int32, batch)
    _need("q", q, dt, batch * cfg.num_q_heads * cfg.head_dim)
    _need("out", out, torch.float32, batch * cfg.num_q_heads * cfg.head_dim)
    _need("workspace", workspace, torch.uint8)
    _need("err", err, torch.int32, 1)
    _cuda(pool, q, page_table, seq_len, out, workspace, err, stream=stream)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cfg.head_dim)
    pool_pages = pool.numel() * 2 // (cfg.num_kv_heads * dense_page_bytes(cfg))
    _check("kvq_decode_attention_dense", load().kvq_decode_attention_dense(
        ctypes.byref(cfg.c()), pool.data_ptr(), pool_pages, q.data_ptr(), batch, page_table.data_ptr(),
        max_pages, seq_len.data_ptr(), float(sm_scale), out.data_ptr(), workspace.data_ptr(),
        workspace.numel(), _ptr(err), _stream(stream)))


def prefill_workspace_bytes(cfg: Config, L: int) -> int:
    return int(load().kvq_prefill_workspace_bytes(ctypes.byref(cfg.c()), L))


def prefill_attention(cfg: Config, q, k, v, out, scores, workspace, sm_scale: float | None = None, stream=None):
    """Causal prefill attention with cumulative attention scores: q [L][Hq][D], k, v
    [L][Hkv][D] (cache dtype), out fp32 [L][Hq][D], scores fp32 [Hkv][L]."""
    dt, D = torch_dtype(cfg.dtype), cfg.head_dim
    L = q.shape[0]
    _need("q", q, dt, L * cfg.num_q_heads * D)
    _need("k", k, dt, L * cfg.num_kv_heads * D)
    _need("v", v, dt, L * cfg.num_kv_heads * D)
    _need("out", out, torch.float32, L * cfg.num_q_heads * D)
    _need("scores", scores, torch.float32, cfg.num_kv_heads * L)
    _need("workspace", workspace, torch.uint8)
    _cuda(q, k, v, out, scores, workspace, stream=stream)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    _check("kvq_prefill_attention", load().kvq_prefill_attention(
        ctypes.byref(cfg.c()), q.data_ptr(), k.data_ptr(), v.data_ptr(), L, float(sm_scale), out.data_ptr(),
        scores.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))


def retain_tokens(cfg: Config, scores, n_heavy: int, n_recent: int, keep, n_keep, stream=None):
    """Heavy hitters plus recent window per KV head: keep int32 [Hkv][L], n_keep int32 [Hkv]."""
    L = scores.shape[-1]
    _need("scores", scores, torch.float32, cfg.num_kv_heads * L)
    _need("keep", keep, torch.int32, cfg.num_kv_heads * L)
    _need("n_keep", n_keep, torch.int32, cfg.num_kv_heads)
    _cuda(scores, keep, n_keep, stream=stream)
    _check("kvq_retain_tokens", load().kvq_retain_tokens(
        ctypes.byref(cfg.c()), scores.data_ptr(), L, n_heavy, n_recent, keep.data_ptr(), n_keep.data_ptr(),
        _stream(stream)))


def gather_tokens(cfg: Config, k, v, keep, n: int, k_out, v_out, err=None, stream=None):
    """k_out[t][h] = k[keep[h][t]][h] (and v) for t < n: [n][Hkv][D] of the cache dtype."""
    dt, H, D = torch_dtype(cfg.dtype), cfg.num_kv_heads, cfg.head_dim
    L = k.shape[0]
    _need("k", k, dt, L * H * D)
    _need("v", v, dt, L * H * D)
    _need("keep", keep, torch.int32, H * L)
    _need("k_out", k_out, dt, n * H * D)
    _need("v_out", v_out, dt, n * H * D)
    _need("err", err, torch.int32, 1)
    _cuda(k, v, keep, k_out, v_out, err, stream=stream)
    _check("kvq_gather_tokens", load().kvq_gather_tokens(
        ctypes.byref(cfg.c()), k.data_ptr(), v.data_ptr(), L, keep.data_ptr(), n, k_out.data_ptr(),
        v_out.data_ptr(), _ptr(err), _stream(stream)))
