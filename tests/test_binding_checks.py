"""The binding's tensor checks (CPU only): the C ABI takes plain pointers, so the binding
refuses tensors of the wrong element type, non-dense tensors and tensors smaller than the
call's extent before anything reaches the library."""
import pytest
import torch

from bit_mixed_precision_channel_b200 import binding as kb

CFG = kb.Config(num_q_heads=8, num_kv_heads=2, page_tokens=32, num_boost=16)
B, MAXP, POOL = 3, 4, 6


def _decode_args(**over):
    H, Hq, P, D = 2, 8, 32, 128
    a = dict(pool=torch.zeros(POOL * H * kb.page_bytes(CFG), dtype=torch.uint8),
             q=torch.zeros(B, Hq, D, dtype=torch.float16),
             page_table=torch.zeros(B, MAXP, dtype=torch.int32),
             num_pages=torch.zeros(B, dtype=torch.int32),
             res_k=torch.zeros(B, H, P, D, dtype=torch.float16),
             res_v=torch.zeros(B, H, P, D, dtype=torch.float16),
             res_len=torch.zeros(B, dtype=torch.int32),
             out=torch.zeros(B, Hq, D, dtype=torch.float32),
             workspace=torch.zeros(kb.decode_workspace_bytes(CFG, B, MAXP), dtype=torch.uint8))
    a.update(over)
    return a


def test_well_formed_cpu_tensors_fail_only_on_the_device_check():
    with pytest.raises(ValueError, match="CUDA tensors"):
        kb.decode_attention(CFG, **_decode_args())


@pytest.mark.parametrize("over,msg", [
    (dict(q=torch.zeros(B, 8, 128, dtype=torch.bfloat16)), "q: dtype"),
    (dict(out=torch.zeros(B, 8, 128, dtype=torch.float16)), "out: dtype"),
    (dict(page_table=torch.zeros(B, MAXP, dtype=torch.int64)), "page_table: dtype"),
    (dict(page_table=torch.zeros(B * MAXP, dtype=torch.int32)), "page_table must have 2"),
    (dict(num_pages=torch.zeros(B - 1, dtype=torch.int32)), "num_pages: 2 elements"),
    (dict(res_k=torch.zeros(B, 2, 16, 128, dtype=torch.float16)), "res_k: "),
    (dict(q=torch.zeros(B, 128, 8, dtype=torch.float16).transpose(1, 2)), "q must be contiguous"),
    (dict(workspace=torch.zeros(64, dtype=torch.int32)), "workspace: dtype"),
])
def test_decode_rejects_bad_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        kb.decode_attention(CFG, **_decode_args(**over))


def test_quantize_rejects_a_source_shorter_than_its_pages():
    x = torch.zeros(2 * 32 - 1, 2, 128, dtype=torch.float16)  # one token short of 2 pages
    pool = torch.zeros(POOL * 2 * kb.page_bytes(CFG), dtype=torch.uint8)
    dst = torch.tensor([0, 1], dtype=torch.int32)
    with pytest.raises(ValueError, match="k source"):
        kb.quantize_pages(CFG, kb.Source.token_major(x, CFG), kb.Source.token_major(x, CFG), dst, pool)
    with pytest.raises(ValueError, match="dst_pages: dtype"):
        kb.quantize_pages(CFG, kb.Source.token_major(x, CFG), kb.Source.token_major(x, CFG), dst.long(), pool)


def test_append_rejects_a_short_window():
    res = torch.zeros(B, 2, 31, 128, dtype=torch.float16)  # P - 1 tokens per window
    tok = torch.zeros(B, 2, 128, dtype=torch.float16)
    with pytest.raises(ValueError, match="res_k"):
        kb.append_token(CFG, tok, tok, res, res, torch.zeros(B, dtype=torch.int32))


class _FakeCuda:
    """Stands in for a CUDA tensor on a machine without a GPU: only what the device
    check reads."""

    def __init__(self, index):
        self.is_cuda = True
        self.device = torch.device("cuda", index)


def test_tensors_of_another_device_are_refused(monkeypatch):
    """A call whose tensors live on a GPU other than the current one is refused on the
    host (the kernels would run on the current GPU with the other GPU's pointers)."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    kb._cuda(_FakeCuda(0), None, _FakeCuda(0))  # one device, the current one: accepted
    with pytest.raises(ValueError, match="current device is cuda:0"):
        kb._cuda(_FakeCuda(1), _FakeCuda(1))
    with pytest.raises(ValueError, match="tensors of one device"):
        kb._cuda(_FakeCuda(0), _FakeCuda(1))

    class _Stream:
        device = torch.device("cuda", 1)

    with pytest.raises(ValueError, match="stream of cuda:1"):
        kb._cuda(_FakeCuda(0), stream=_Stream())
