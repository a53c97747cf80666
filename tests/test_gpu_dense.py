"""GPU parity of decode attention over an unquantized paged cache (the full-precision
comparison point of the 2-bit cache, on the same kernel and work line): within the
method's tolerance of the oracle's exact fp64 attention over the raw tokens, for ragged
lengths (partial last pages, empty and one-token sequences) and shuffled pages."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import binding as kb
from bit_mixed_precision_channel_b200 import synthetic as syn

from _kv import assert_attention_close, ocfg, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gqa,dtype,P,lens", [
    (4, kb.F16, 128, [4096 + 77, 0, 1, 300]),
    (8, kb.BF16, 128, [2048 + 5, 130]),
    (1, kb.F16, 32, [256, 250, 31]),
    (2, kb.BF16, 64, [64 * 9 + 63, 17]),
])
def test_dense_decode_matches_exact_attention(gqa, dtype, P, lens):
    rng = np.random.default_rng(gqa * 10 + dtype + P)
    H, D = 2, 128
    cfg = kb.Config(num_q_heads=gqa * H, num_kv_heads=H, page_tokens=P, num_boost=16, dtype=dtype)
    B = len(lens)
    max_pages = max(1, max((L + P - 1) // P for L in lens))
    n_used = sum((L + P - 1) // P for L in lens)
    pool_pages = n_used + 3
    order = rng.permutation(pool_pages)
    pool = np.zeros((pool_pages, H, 2, P, D), np.uint16)
    table = np.full((B, max_pages), -1, np.int32)
    raw = []
    nxt = 0
    for b, L in enumerate(lens):
        sig = np.exp(rng.standard_normal((H, D))).astype(np.float32) * 2
        K = syn.to_bits(rng.standard_normal((L, H, D)).astype(np.float32) * sig, dtype)
        V = syn.to_bits(rng.standard_normal((L, H, D)).astype(np.float32), dtype)
        raw.append((K, V))
        for i in range((L + P - 1) // P):
            pg = int(order[nxt])
            nxt += 1
            table[b, i] = pg
            n = min(P, L - i * P)
            pool[pg, :, 0, :n] = K[i * P:i * P + n].transpose(1, 0, 2)
            pool[pg, :, 1, :n] = V[i * P:i * P + n].transpose(1, 0, 2)
    q = syn.to_bits(rng.standard_normal((B, gqa * H, D)).astype(np.float32), dtype)
    dpool = to_dev(pool.reshape(-1), dtype)
    ws = torch.zeros(kb.decode_workspace_bytes(cfg, B, max_pages), dtype=torch.uint8, device="cuda")
    out = torch.full((B, gqa * H, D), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb.decode_attention_dense(cfg, dpool, to_dev(q, dtype), torch.from_numpy(table).cuda(),
                              torch.tensor(lens, dtype=torch.int32, device="cuda"), out, ws, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    oc = ocfg(cfg)
    empty_pool = np.zeros((1, H, oc.record_bytes), np.uint8)
    for b, L in enumerate(lens):
        K, V = raw[b]
        for h in range(H):
            want = oracle.decode_unit(empty_pool, oc, h, [], K[:, h], V[:, h], q[b, h * gqa:(h + 1) * gqa],
                                      1.0 / math.sqrt(D))
            assert_attention_close(got[b, h * gqa:(h + 1) * gqa], want, f"seq {b} (len {L}) kv head {h}")
    assert not ws[-4 * B * H:].any()  # arrival counters back to zero
