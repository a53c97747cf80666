"""CPU checks of the C-ABI library: it loads, exports every function include/kvq.h
declares, and its host-side checks (no GPU involved) behave as documented."""
import ctypes
import os
import re
import subprocess

import pytest

from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "kvq.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kb.load()


def test_header_declares_the_expected_calls():
    names = _declared()
    for n in ["kvq_select_boost_channels", "kvq_quantize_page_keys", "kvq_quantize_values",
              "kvq_quantize_pages", "kvq_append_token", "kvq_flush_residual", "kvq_append_flush", "kvq_decode_attention",
              "kvq_decode_workspace_bytes", "kvq_page_layout", "kvq_page_bytes", "kvq_check_config",
              "kvq_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", kb.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)
    # only the C ABI is exported (the build hides everything else)
    assert all(n.startswith("kvq_") or not n.startswith("_Z") for n in exported)


def test_layout_matches_hand_worked_sizes(lib):
    cfg = kb.Config(num_q_heads=32, num_kv_heads=8, page_tokens=128, num_boost=32)
    L = kb.page_layout(cfg)
    assert L["payload_bytes"] == 12064 and L["record_bytes"] == 12160
    assert kb.page_bytes(kb.Config(page_tokens=32, num_boost=16, num_q_heads=1, num_kv_heads=1)) == 2944


@pytest.mark.parametrize("over,status", [
    (dict(head_dim=64), 2), (dict(num_q_heads=12, num_kv_heads=8), 1), (dict(num_q_heads=48, num_kv_heads=4), 2),
    (dict(page_tokens=96), 2), (dict(page_tokens=100), 1), (dict(key_group=64), 2), (dict(num_boost=8), 1),
    (dict(num_boost=144), 1), (dict(num_boost=48), 2), (dict(num_boost=64), 0), (dict(key_bits=3), 2), (dict(dtype=7), 2), (dict(), 0), (dict(num_boost=0), 0),
])
def test_check_config(lib, over, status):
    assert kb.check_config(kb.Config(**over)) == status


def test_calls_reject_bad_arguments_before_any_launch(lib):
    cfg = kb.Config()
    c = ctypes.byref(cfg.c())
    # null pointers / negative sizes -> KVQ_ERR_INVALID_ARG, without touching a device
    assert lib.kvq_append_token(c, 4, None, None, None, None, None, None, None) == 1
    assert lib.kvq_append_token(c, -1, 16, 16, 16, 16, 16, None, None) == 1
    assert lib.kvq_append_token(c, 0, None, None, None, None, None, None, None) == 0
    src = kb._Source(None, 0, 0, 0)
    assert lib.kvq_quantize_pages(c, src, src, None, 3, None, 1, None, None) == 1
    assert lib.kvq_quantize_pages(c, src, src, None, 0, None, 1, None, None) == 0
    misaligned = kb._Source(0x1008, 128 * 8 * 128, 8 * 128, 128)
    assert lib.kvq_quantize_pages(c, misaligned, misaligned, 0x100, 1, 0x1000, 1, None, None) == 1
    odd_stride = kb._Source(0x1000, 128 * 8 * 128, 8 * 128 + 1, 128)
    assert lib.kvq_quantize_pages(c, odd_stride, odd_stride, 0x100, 1, 0x1000, 1, None, None) == 1
    assert lib.kvq_flush_residual(c, 2, None, None, None, None, None, 4, None, None, 1, None, None) == 1
    p16 = 0x1000
    assert lib.kvq_append_flush(c, 2, p16, p16, p16, p16, p16, p16, p16, 4, p16, p16, 1, None, None, None,
                                None) == 1  # no counters
    assert lib.kvq_append_flush(c, 2, p16 + 8, p16, p16, p16, p16, p16, p16, 4, p16, p16, 1, None, p16, None,
                                None) == 1  # misaligned token
    assert lib.kvq_append_flush(c, 0, None, None, None, None, None, None, None, 4, None, None, 1, None, None,
                                None, None) == 0
    assert lib.kvq_decode_attention(c, None, 1, None, 2, None, 4, None, None, None, None, 0.1, None, None, 0,
                                    None, None) == 1
    # workspace smaller than kvq_decode_workspace_bytes -> KVQ_ERR_CAPACITY
    need = lib.kvq_decode_workspace_bytes(c, 2, 4)
    assert need > 0
    p = 0x10000
    assert lib.kvq_decode_attention(c, p, 1, p, 2, p, 4, p, p, p, p, 0.1, p, p, need - 1, None, None) == 4
    # unsupported config is reported before pointers are looked at
    bad = ctypes.byref(kb.Config(head_dim=256).c())
    assert lib.kvq_decode_attention(bad, None, 1, None, 2, None, 4, None, None, None, None, 0.1, None, None, 0,
                                    None, None) == 2


def test_prefill_workspace_holds_two_values_per_query_row(lib):
    """The prefill workspace holds each query row's log2-sum-exp and each query head's
    cumulative scores: 2 * Hq * L fp32, rounded up to 256 bytes; 0 for a bad config."""
    cfg = kb.Config(num_q_heads=32, num_kv_heads=8, page_tokens=128, num_boost=32)
    for L in (1, 255, 4096):
        assert kb.prefill_workspace_bytes(cfg, L) == (2 * 32 * L * 4 + 255) // 256 * 256
    assert lib.kvq_prefill_workspace_bytes(ctypes.byref(kb.Config(head_dim=64).c()), 16) == 0


def test_status_strings(lib):
    for s in range(5):
        assert kb.status_string(s)
    assert kb.status_string(99) == "unknown status"
