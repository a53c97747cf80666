"""bench.py's JSON contract on the CPU: the reference arm (the oracle on the host cores)
prints the library arm's metric, unit and config, with its own cpu_baseline and e2e
objects, and the config object names the workload and its L2 footprint."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_mixed_precision_channel_b200 import binding as kb  # noqa: E402
from bit_mixed_precision_channel_b200 import synthetic as syn  # noqa: E402


def _payload(w):
    cfg = kb.Config(head_dim=w.D, num_q_heads=w.Hq, num_kv_heads=w.Hkv, page_tokens=w.P, key_group=w.G,
                    num_boost=w.k, dtype=w.dtype)
    return kb.page_layout(cfg)["payload_bytes"]


def test_workload_config_names_the_workload_and_scales_with_ranks():
    w = syn.WORKLOADS[bench.WORKLOAD]
    one = bench.workload_config(w, 32, 1, _payload(w))
    two = bench.workload_config(w, 32, 2, _payload(w))
    assert one["global_batch"] == w.batch and two["global_batch"] == 2 * w.batch
    assert one["parallelism"] == "single GPU" and two["parallelism"] == "replicas x2"
    assert one["seq_len"] == w.context and one["layers"] == 32
    assert "Llama-3-8B-shaped" in one["workload"] and "larger than L2" in one["l2"]
    # 32 layer caches of packed pages are far above the 126 MB L2
    gb = float(one["l2"].split("caches, ")[1].split(" GB")[0])
    assert gb * 1e9 > 4 * 126e6


def test_reference_arm_prints_the_library_arms_contract():
    args = type("A", (), {"warmup": 0, "steps": 1, "gpus": 1, "layers": 32})()
    r = bench.run_reference(args)
    w = syn.WORKLOADS[bench.WORKLOAD]
    assert r["impl"] == "reference"
    assert r["metric"] == bench.METRIC and r["unit"] == "GB/s" and r["higher_is_better"] is True
    assert r["config"] == bench.workload_config(w, 32, 1, _payload(w))
    assert r["value"] > 0 and r["steps"] == 1 and r["warmup"] == 0
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == r["value"] and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_off_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"warmup": 0, "steps": 1, "gpus": 2, "layers": 32})()
    assert bench.run_reference(args) is None


@pytest.mark.parametrize("res", [0, 57])
def test_decode_bytes_count_pages_residual_query_output_and_table(res):
    w = syn.WORKLOADS[bench.WORKLOAD]
    payload = _payload(w)
    n_pages = w.context // w.P
    got = bench.decode_bytes(w, payload, n_pages, res)
    want = (w.batch * w.Hkv * n_pages * payload            # packed pages
            + w.batch * w.Hkv * res * 2 * w.D * 2          # residual K and V rows
            + w.batch * w.Hq * w.D * 2                     # q
            + w.batch * w.Hq * w.D * 4                     # fp32 output
            + w.batch * n_pages * 4                        # page-table entries
            + w.batch * 8)                                 # num_pages and res_len
    assert got == want
