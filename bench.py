"""Benchmark of the 2-bit mixed-precision KV cache decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

Workload (one GPU): the Llama-3-8B-shaped decode layer — batch 16, 32 query / 8 KV
heads, head_dim 128, 4096-token prompts in pages of 128, 32 boosted key channels of
128 (25%), fp16 — replicated over 32 layers, as a decode step of that model walks its
32 layers.  The 32 layer caches (1.6 GB of packed KV) are far larger than the 126 MB
L2, so every step reads its pages from HBM.  Inputs are seeded synthetic tensors
(see bit_mixed_precision_channel_b200/synthetic.py).

A step = for every layer: append the new token to the residual window, flush full
windows, decode attention over pages + window (all rows of the hot path; the prompt
pages were quantized once at prefill, whose rate is reported as "quantize").  The host
tracks the windows' lengths, so the flush is launched only on steps where a window
fills (once every 128 steps; "flush_steps" counts them in the timed region, and the
flush rate of the ragged workload is reported under configs).  Each kind of step
(without / with flush) is captured once in a CUDA graph and replayed.

value: decode-attention algorithmic bytes of all layers / step time (GB/s), whole job
(summed over ranks for N > 1, each rank running its own batch: weak scaling).
roofline: the decode kernel alone, timed over L launches per replay in its own loop.
e2e: the same step driven from host buffers: q, k_new, v_new copied in from pinned
memory and the output copied back, inside the timed region.
cpu_baseline / --impl reference: the CPU oracle (oracle/, fp64 attention) timed on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOAD = "llama3_8b"
# DRAM traffic of one decode launch of this workload (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture of the decode kernel), valid only for the
# kernel source it was taken on: the bench reports it while the decode kernel source
# still hashes to this value.
DECODE_TRAFFIC = {"source_sha256": "0207a5f1d55e37f879fe053e08a049bbf13c710e2b7c307fb8b730a1a0cfdd68",
                  "bytes": 50298880 + 22528}
LAYERS = 32
METRIC = "2-bit KV decode-attn GB/s & % of HBM peak; quantize tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload measurements")
    ap.add_argument("--leg", default="main",
                    help="main (the contract line), minikv (the MiniKV prefill leg alone), or "
                         "decode:<workload> (one full-size cache, 5 decode launches: a short program "
                         "for profiling one workload's decode kernel)")
    return ap.parse_args()


def peak_tensor():
    """Measured dense bf16 tensor throughput (TFLOP/s, burst), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ workload bytes

def decode_traffic():
    """ncu DRAM bytes per decode launch, or None once the kernel source has changed."""
    import hashlib
    src = os.path.join(ROOT, "bit_mixed_precision_channel_b200", "csrc", "kvq_decode_impl.cuh")
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    return DECODE_TRAFFIC["bytes"] if digest == DECODE_TRAFFIC["source_sha256"] else None


def max_over_ranks(times_ms, device, world):
    """Per-rank times -> the maximum over all ranks (one all-reduce MAX; no-op at N = 1)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(times_ms, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_gbs(world, bytes_per_rank, ms):
    """Whole-job throughput: every rank moves bytes_per_rank in the slowest rank's time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def decode_bytes(w, payload, n_pages, res_len):
    """Algorithmic bytes of one decode-attention launch (one layer): packed pages
    (codes + scales + zeros + boost indices), the fp16 residual K and V, the query,
    the fp32 output, the page table entries and the two lengths of every sequence."""
    B, Hkv, Hq, D = w.batch, w.Hkv, w.Hq, w.D
    return (B * Hkv * n_pages * payload + B * Hkv * res_len * 2 * D * 2 + B * Hq * D * 2 + B * Hq * D * 4
            + 4 * B * n_pages + 8 * B)


# ------------------------------------------------------------------ clocks during timing

_CLOCK_POLLER = r"""
import sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
out = open(sys.argv[2], "w")
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
while True:
    try:
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        out.write(f"{time.time():.4f} {sm} {mx} {r}\n"); out.flush()
    except Exception as e:
        out.write(f"# {e}\n"); out.flush()
    time.sleep(0.002)
"""

REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
           0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle", 0x2: "applications_clocks_setting",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, uuid: str):
        self.path = tempfile.mktemp(prefix="kvq_clocks_", suffix=".txt")
        self.proc = subprocess.Popen([sys.executable, "-c", _CLOCK_POLLER, uuid, self.path],
                                     stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        self.t0 = self.t1 = None

    def wait_ready(self, timeout=20.0):
        t = time.time()
        while time.time() - t < timeout:
            if os.path.exists(self.path) and os.path.getsize(self.path) > 0:
                return True
            time.sleep(0.05)
        return False

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    if line.startswith("#"):
                        continue
                    t, sm, mx, r = line.split()
                    rows.append((float(t), int(sm), int(mx), int(r)))
            os.unlink(self.path)
        except OSError:
            pass
        sel = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": rows[0][2] if rows else None, "reasons": [], "samples": 0}
        mask = 0
        for r in sel:
            mask |= r[3]
        reasons = [name for bit, name in REASONS.items() if mask & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(r[1] for r in sel), "sm_max_mhz": sel[0][2], "reasons": reasons,
                "samples": len(sel)}


# ------------------------------------------------------------------ CPU oracle baseline

def cpu_baseline(w, K, V, res_k_host, res_v_host, res_len, q_host, budget_s=12.0, threads=None):
    """The oracle (oracle/, plain C, fp64 attention) on the host cores: decode attention
    of whole units (sequence, kv head) of one layer, repeated over the units of the
    step until ~budget_s of wall time; returns GB/s over the same algorithmic bytes."""
    import concurrent.futures as cf

    import oracle

    oc = oracle.Cfg(D=w.D, Hq=w.Hq, Hkv=w.Hkv, P=w.P, G=w.G, k=w.k, dtype=w.dtype)
    P = w.P
    n_pages = K.shape[1] // P
    payload = oracle.layout(P, w.D, w.k, w.G)["payload_bytes"]
    threads = threads or max(1, min(os.cpu_count() or 1, 32))
    units = [(b, h) for b in range(w.batch) for h in range(w.Hkv)]
    pools = {}

    def quant(b):
        pool = np.zeros((n_pages, w.Hkv, oc.record_bytes), np.uint8)
        for i in range(n_pages):
            for h in range(w.Hkv):
                pool[i, h] = oracle.quantize_page(K[b, i * P:(i + 1) * P, h], V[b, i * P:(i + 1) * P, h], oc)
        return b, pool

    with cf.ThreadPoolExecutor(threads) as ex:
        for b, pool in ex.map(quant, range(w.batch)):
            pools[b] = pool
    g = w.gqa
    sm = 1.0 / math.sqrt(w.D)

    def unit(bh):
        b, h = bh
        return oracle.decode_unit(pools[b], oc, h, list(range(n_pages)), res_k_host[b, h, :res_len],
                                  res_v_host[b, h, :res_len], q_host[b, h * g:(h + 1) * g], sm)

    per_unit = payload * n_pages + res_len * 2 * w.D * 2 + g * w.D * 6 + 4 * n_pages
    done = 0
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(threads) as ex:
        while time.perf_counter() - t0 < budget_s:
            list(ex.map(unit, units))
            done += len(units)
    dt = time.perf_counter() - t0
    return {"value": per_unit * done / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} (sequence, kv head) decode units of one layer ({done // len(units)} full "
                      f"passes over the {len(units)} units), fp64 attention over {n_pages} pages + "
                      f"{res_len} residual tokens each, {dt:.1f} s on {threads} threads"}


# ------------------------------------------------------------------ GPU benchmark

def run_gpu(args):
    import torch
    import torch.distributed as dist

    from bit_mixed_precision_channel_b200 import binding as kb
    from bit_mixed_precision_channel_b200 import synthetic as syn
    from bit_mixed_precision_channel_b200.cache import PagedKVCache

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = syn.WORKLOADS[WORKLOAD]
    L_layers = args.layers
    cfg = kb.Config(head_dim=w.D, num_q_heads=w.Hq, num_kv_heads=w.Hkv, page_tokens=w.P, key_group=w.G,
                    num_boost=w.k, dtype=w.dtype)
    B, P, D = w.batch, w.P, w.D
    n_pages = w.context // P
    total_steps = args.warmup + args.steps + 3
    max_pages = n_pages + total_steps // P + 2
    pool_pages = B * max_pages
    payload = kb.page_layout(cfg)["payload_bytes"]
    tdt = kb.torch_dtype(w.dtype)

    def dev_bits(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).to(dev)

    # -------- prompts (the same synthetic prompt for every layer replica; each layer has its own cache)
    sigma = syn.key_channel_sigma(w)
    Kh = np.stack([syn.keys(w, b + 1000 * rank, 0, w.context, sigma) for b in range(B)])
    Vh = np.stack([syn.values(w, b + 1000 * rank, 0, w.context) for b in range(B)])
    Kd, Vd = dev_bits(Kh), dev_bits(Vh)
    caches = [PagedKVCache(cfg, B, max_pages, pool_pages, device=dev) for _ in range(L_layers)]

    # quantize leg: prefill of every layer (page allocation and tables untimed), then the
    # quantize launches of all layers timed: one launch per layer quantizes its 16 x 4096
    # tokens into the pages the prefill assigned (the same records again)
    for c in caches:
        c.prefill_batch(Kd, Vd)
    n_seq_pages = w.context // P
    srcK = kb.Source.token_major(Kd.view(B * w.context, w.Hkv, D), cfg)
    srcV = kb.Source.token_major(Vd.view(B * w.context, w.Hkv, D), cfg)
    dsts = [c.page_table[:, :n_seq_pages].contiguous().view(-1) for c in caches]
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for c, dst in zip(caches, dsts):
        kb.quantize_pages(cfg, srcK, srcV, dst, c.pool, c.err)
    e1.record()
    torch.cuda.synchronize()
    q_ms = e0.elapsed_time(e1) / L_layers
    quant_tokens_per_s = B * w.context / (q_ms * 1e-3)
    quant_bytes = B * w.context * w.Hkv * D * 2 * 2 + B * n_pages * w.Hkv * payload
    for c in caches:
        assert c.check_errors() == 0

    # -------- per-layer decode inputs (static buffers the graph reads)
    kn, vn = syn.step_tokens(w, 0, sigma)
    qh = syn.queries(w, 0)
    qs = [dev_bits(qh) for _ in range(L_layers)]
    kns = [dev_bits(kn) for _ in range(L_layers)]
    vns = [dev_bits(vn) for _ in range(L_layers)]
    outs = [torch.empty(B, w.Hq, D, device=dev) for _ in range(L_layers)]

    def device_step(flush):
        # the host knows which windows fill this step: the flush runs only then
        for i, c in enumerate(caches):
            c.append(kns[i], vns[i])
            if flush:
                c.flush()
            c.attend(qs[i], outs[i])

    def attend_only():
        for i, c in enumerate(caches):
            c.attend(qs[i], outs[i])

    def host_step(flag_list):
        for i, c in enumerate(caches):
            flag_list[i] = c.reserve_flush_pages()

    def host_commit(flag_list):
        for i, c in enumerate(caches):
            c.commit_host(flag_list[i])

    def flushing(flag_list):
        return any(len(f) > 0 for f in flag_list)

    flags = [None] * L_layers
    # eager warm-up (also sets kernel attributes before capture)
    for _ in range(2):
        host_step(flags)
        device_step(True)
        host_commit(flags)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    # one graph per step kind: without and with the flush of full windows
    g_step = {False: torch.cuda.CUDAGraph(), True: torch.cuda.CUDAGraph()}
    g_attn = torch.cuda.CUDAGraph()
    for fl, graph in g_step.items():
        with torch.cuda.graph(graph, stream=stream):
            device_step(fl)
    with torch.cuda.graph(g_attn, stream=stream):
        attend_only()
    # e2e: host buffers in pinned memory, copies inside the graph
    q_pin = [torch.from_numpy(qh.view(np.int16)).view(tdt).pin_memory() for _ in range(L_layers)]
    kn_pin = [torch.from_numpy(kn.view(np.int16)).view(tdt).pin_memory() for _ in range(L_layers)]
    vn_pin = [torch.from_numpy(vn.view(np.int16)).view(tdt).pin_memory() for _ in range(L_layers)]
    out_pin = [torch.empty(B, w.Hq, D).pin_memory() for _ in range(L_layers)]
    # The copies run on two copy streams forked inside the graph: every layer's inputs go
    # up in layer order while earlier layers compute, and every layer's output comes back
    # while later layers compute.  Each step still moves all inputs and all outputs.
    g_e2e = {False: torch.cuda.CUDAGraph(), True: torch.cuda.CUDAGraph()}
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    for fl, graph in g_e2e.items():
        with torch.cuda.graph(graph, stream=stream):
            start = torch.cuda.Event()
            start.record(stream)
            up.wait_event(start)
            down.wait_event(start)
            landed, done = [], []
            with torch.cuda.stream(up):
                for i in range(L_layers):
                    qs[i].copy_(q_pin[i], non_blocking=True)
                    kns[i].copy_(kn_pin[i], non_blocking=True)
                    vns[i].copy_(vn_pin[i], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(up)
                    landed.append(ev)
            for i, c in enumerate(caches):
                stream.wait_event(landed[i])
                c.append(kns[i], vns[i])
                if fl:
                    c.flush()
                c.attend(qs[i], outs[i])
                ev = torch.cuda.Event()
                ev.record(stream)
                done.append(ev)
            with torch.cuda.stream(down):
                for i in range(L_layers):
                    down.wait_event(done[i])
                    out_pin[i].copy_(outs[i], non_blocking=True)
            stream.wait_stream(down)
            stream.wait_stream(up)
    h2d_bytes = L_layers * (qh.nbytes + kn.nbytes + vn.nbytes)
    d2h_bytes = L_layers * B * w.Hq * D * 4

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(graph, n, warm, advance):
        # graph: one graph, or (advance) a dict of the step graphs without / with flush
        for _ in range(warm):
            if advance:
                host_step(flags)
                graph[flushing(flags)].replay()
                host_commit(flags)
            else:
                graph.replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            if advance:
                host_step(flags)
                graph[flushing(flags)].replay()
                host_commit(flags)
            else:
                graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return a.elapsed_time(b) / n  # ms per replay

    def snapshot():
        return ([c.res_len.clone() for c in caches], [list(c.host_res_len) for c in caches])

    def restore(s):
        for c, r, h in zip(caches, s[0], s[1]):
            c.res_len.copy_(r)
            c.host_res_len = list(h)

    snap = snapshot()
    res0 = caches[0].host_res_len[0]
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    clocks.wait_ready()
    with torch.cuda.stream(stream):
        # main timed region: K decode steps over all layers
        for _ in range(args.warmup):
            host_step(flags)
            g_step[flushing(flags)].replay()
            host_commit(flags)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        clocks.mark_start()
        ev_a, ev_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev_a.record(stream)
        flush_steps = 0
        for _ in range(args.steps):
            host_step(flags)
            fl = flushing(flags)
            flush_steps += fl
            g_step[fl].replay()
            host_commit(flags)
        ev_b.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
        barrier()
        step_ms = ev_a.elapsed_time(ev_b) / args.steps
    clock_info = clocks.stop()
    res_avg = res0 + args.warmup + (args.steps - 1) / 2 + 1  # residual length during the timed steps
    res_end = caches[0].host_res_len[0]
    for c in caches:
        assert c.check_errors() == 0, "device error flags set"

    with torch.cuda.stream(stream):
        attn_ms = timed(g_attn, max(args.steps, 20), 3, advance=False) / L_layers
        restore(snap)
        e2e_ms = timed(g_e2e, args.steps, args.warmup, advance=True)
    restore(snap)

    bytes_step = L_layers * decode_bytes(w, payload, n_pages, res_avg)
    bytes_attn = decode_bytes(w, payload, n_pages, res_end)
    step_ms, e2e_ms, attn_ms = max_over_ranks([step_ms, e2e_ms, attn_ms], dev, world)
    peak, peak_kind = peaks()
    value = whole_job_gbs(world, bytes_step, step_ms)
    e2e_value = whole_job_gbs(world, bytes_step, e2e_ms)
    achieved = bytes_attn / (attn_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": workload_config(w, L_layers, world, payload),
        "hbm_frac": round(value / world / peak, 4),
        "quantize": {"tokens_per_s": round(quant_tokens_per_s, 1), "ms_per_layer": round(q_ms, 4),
                     "gbs": round(quant_bytes / (q_ms * 1e-3) / 1e9, 1),
                     "what": f"prefill of {B} x {w.context} tokens into pages (select + keys + values), per layer"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": decode_traffic(),
                     "kernel": "decode_kernel<__half,4>", "peak_source": peak_kind,
                     "per_launch_bytes": bytes_attn, "ms_per_launch": round(attn_ms, 5)},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes, "ms_per_step": round(e2e_ms, 4)},
        # append and decode per layer; flush and commit per layer on steps where windows fill
        "gpu_launches": args.steps * L_layers * 2 + flush_steps * L_layers * 2,
        "flush_steps": flush_steps,
        "clocks": clock_info,
    }
    if world == 1 and not args.no_configs:
        cfgs = {WORKLOAD: {"decode_us_per_launch": round(attn_ms * 1e3, 2), "decode_gbs": round(achieved, 1),
                           "frac": round(achieved / peak, 4), "bytes_per_launch": bytes_attn,
                           "replicas": L_layers, "quantize_tokens_per_s": round(quant_tokens_per_s, 1),
                           "quantize_gbs": result["quantize"]["gbs"]}}
        cfgs[WORKLOAD + "_l2_flushed"] = l2_flushed_single(dev, peak)
        cfgs["qwen3_8b_long"] = workload_bench("qwen3_8b_long", dev, peak)
        cfgs["llama3_70b_batch"] = workload_bench("llama3_70b_batch", dev, peak)
        cfgs["ragged_serving"] = workload_bench("ragged_serving", dev, peak, flush_steps=256)
        result["configs"] = cfgs
        result["vs_fp16_dense"] = compare_dense(dev, peak)
        result["minikv_prefill"] = prefill_bench(dev, peak_tensor())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # every step appended the same k_new / v_new, so the windows hold copies of them
        rk = np.repeat(kn[:, :, None, :], res_end, axis=2)
        rv = np.repeat(vn[:, :, None, :], res_end, axis=2)
        result["cpu_baseline"] = cpu_baseline(w, Kh, Vh, rk, rv, res_end, qh)
    if world > 1:
        dist.barrier()
        del g_step, g_attn, g_e2e, graph
        dist.destroy_process_group()
    return result if rank == 0 else None


# ------------------------------------------------------------------ the other workloads

def _device_prompts(w, lens, sigma_dev, gen, tdt, dev):
    """Seeded synthetic prompts drawn on the device with the workload's distributions
    (keys N(0,1) x per-channel sigma, values N(0,1)); the values differ from the numpy
    streams the parity tests use, the distributions do not."""
    for b, L in enumerate(lens):
        K = (torch_randn((int(L), w.Hkv, w.D), gen, dev) * sigma_dev).to(tdt)
        V = torch_randn((int(L), w.Hkv, w.D), gen, dev).to(tdt)
        yield b, K, V


def torch_randn(shape, gen, dev):
    import torch
    return torch.randn(shape, generator=gen, device=dev)


def workload_bench(name, dev, peak, min_bytes=512e6, flush_steps=0, iters=20):
    """Decode attention (and quantize) throughput of one workload on one GPU.
    Replicas of the layer cache are added until the packed pages exceed min_bytes (four
    times the L2), and the decode launches cycle through them."""
    import torch

    from bit_mixed_precision_channel_b200 import binding as kb
    from bit_mixed_precision_channel_b200 import synthetic as syn
    from bit_mixed_precision_channel_b200.cache import PagedKVCache

    w = syn.WORKLOADS[name]
    cfg = kb.Config(head_dim=w.D, num_q_heads=w.Hq, num_kv_heads=w.Hkv, page_tokens=w.P, key_group=w.G,
                    num_boost=w.k, dtype=w.dtype)
    tdt = kb.torch_dtype(w.dtype)
    lens = syn.lengths(w)
    B, P, H = w.batch, w.P, w.Hkv
    payload = kb.page_layout(cfg)["payload_bytes"]
    page_bytes = int(sum(lens // P)) * H * payload
    # replicas cycle through identical lengths; the flush steps run on a single cache
    replicas = 1 if flush_steps else max(1, math.ceil(min_bytes / page_bytes))
    max_pages = int(max(lens) // P + flush_steps // P + 2)
    pool_pages = int(sum(lens // P) + B * (flush_steps // P + 2))
    sigma = torch.from_numpy(syn.key_channel_sigma(w)).to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    caches = []
    q_ms = 0.0
    for r in range(replicas):
        c = PagedKVCache(cfg, B, max_pages, pool_pages, device=dev, page_order=syn.page_order(w, pool_pages))
        full_k, full_v, dsts = [], [], []
        for b, K, V in _device_prompts(w, lens, sigma, gen, tdt, dev):
            c.prefill(b, K, V)
            n = int(lens[b]) // P
            if r == 0 and n:
                full_k.append(K[:n * P])
                full_v.append(V[:n * P])
                dsts += c.host_pages[b][:n]
        if r == 0:
            # quantize: every full page of the workload in one launch, into the pages the
            # prefill assigned (the same records again)
            fk, fv = torch.cat(full_k), torch.cat(full_v)
            dst = torch.tensor(dsts, dtype=torch.int32, device=dev)
            srck, srcv = kb.Source.token_major(fk, cfg), kb.Source.token_major(fv, cfg)
            for _ in range(2):
                kb.quantize_pages(cfg, srck, srcv, dst, c.pool, c.err)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(5):
                kb.quantize_pages(cfg, srck, srcv, dst, c.pool, c.err)
            e1.record()
            torch.cuda.synchronize()
            q_ms = e0.elapsed_time(e1) / 5
            n_tok = int(fk.shape[0])
            del fk, fv, full_k, full_v
        caches.append(c)
    q = (torch_randn((B, w.Hq, w.D), gen, dev)).to(tdt)
    out = torch.empty(B, w.Hq, w.D, device=dev)
    res = {}
    # flush rate (ragged serving): eager decode steps, the flush calls timed alone
    if flush_steps:
        c = caches[0]
        kn = (torch_randn((B, H, w.D), gen, dev) * sigma).to(tdt)
        vn = torch_randn((B, H, w.D), gen, dev).to(tdt)
        flushed, f_ms = 0, 0.0
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(flush_steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for s in range(flush_steps):
            fl = c.reserve_flush_pages()
            c.append(kn, vn)
            ev[s][0].record()
            c.flush()
            ev[s][1].record()
            c.attend(q, out)
            c.commit_host(fl)
            flushed += len(fl)
        t1.record()
        torch.cuda.synchronize()
        f_ms = sum(a.elapsed_time(b) for a, b in ev)
        res["flush"] = {"steps": flush_steps, "flushed_pages": flushed * H, "flush_ms_total": round(f_ms, 3),
                        "flush_ms_per_step": round(f_ms / flush_steps, 4),
                        "flushed_page_heads_per_s": round(flushed * H / (f_ms * 1e-3), 1),
                        "step_ms_eager": round(t0.elapsed_time(t1) / flush_steps, 4),
                        "what": "append + flush + attend per step; the flush calls (quantize of full "
                                "windows + page-table commit) timed with events around them"}
        assert c.check_errors() == 0
    for c in caches:
        c.attend(q, out)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in caches:
            c.attend(q, out)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
    ms = a.elapsed_time(b) / iters / replicas
    c = caches[0]
    nps = c.num_pages.cpu().numpy().astype(np.int64)
    rls = c.res_len.cpu().numpy().astype(np.int64)
    nbytes = int(H * (nps * payload).sum() + H * rls.sum() * 2 * w.D * 2 + B * w.Hq * w.D * (2 + 4)
                 + 4 * nps.sum() + 8 * B)
    for c in caches:
        assert c.check_errors() == 0
    res.update({"decode_us_per_launch": round(ms * 1e3, 2), "decode_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4), "bytes_per_launch": nbytes,
                "replicas": replicas, "tokens": int(lens.sum()),
                "quantize_tokens_per_s": round(n_tok / (q_ms * 1e-3), 1),
                "quantize_gbs": round((n_tok * H * w.D * 2 * 2 + (n_tok // P) * H * payload) / (q_ms * 1e-3) / 1e9, 1),
                "quantize_ms": round(q_ms, 4)})
    del caches, g
    torch.cuda.empty_cache()
    return res


def l2_flushed_single(dev, peak, iters=20):
    """Config 2 with one layer cache (50 MB, inside the L2) and a 512 MB read between the
    timed launches, outside the timed region, so every launch reads from HBM (a read
    leaves clean lines: no write-back competes with the timed launch)."""
    import torch

    from bit_mixed_precision_channel_b200 import binding as kb
    from bit_mixed_precision_channel_b200 import synthetic as syn
    from bit_mixed_precision_channel_b200.cache import PagedKVCache

    w = syn.WORKLOADS[WORKLOAD]
    cfg = kb.Config(head_dim=w.D, num_q_heads=w.Hq, num_kv_heads=w.Hkv, page_tokens=w.P, key_group=w.G,
                    num_boost=w.k, dtype=w.dtype)
    tdt = kb.torch_dtype(w.dtype)
    B, P, H = w.batch, w.P, w.Hkv
    payload = kb.page_layout(cfg)["payload_bytes"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    sigma = torch.from_numpy(syn.key_channel_sigma(w)).to(dev)
    c = PagedKVCache(cfg, B, w.context // P + 2, B * (w.context // P + 2), device=dev)
    K = (torch_randn((B, w.context, H, w.D), gen, dev) * sigma).to(tdt)
    V = torch_randn((B, w.context, H, w.D), gen, dev).to(tdt)
    c.prefill_batch(K, V)
    del K, V
    q = torch_randn((B, w.Hq, w.D), gen, dev).to(tdt)
    out = torch.empty(B, w.Hq, w.D, device=dev)
    scrub = torch.ones(128 << 20, dtype=torch.float32, device=dev)  # 512 MB
    sink = torch.empty(1, device=dev)
    for _ in range(3):
        c.attend(q, out)
    tot = 0.0
    for _ in range(iters):
        torch.sum(scrub, dim=0, keepdim=True, out=sink)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        c.attend(q, out)
        b.record()
        torch.cuda.synchronize()
        tot += a.elapsed_time(b)
    ms = tot / iters
    nbytes = B * H * (w.context // P) * payload + B * w.Hq * w.D * 6 + 4 * B * (w.context // P) + 8 * B
    assert c.check_errors() == 0
    return {"decode_us_per_launch": round(ms * 1e3, 2), "decode_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4), "bytes_per_launch": nbytes,
            "what": "one layer cache, a 512 MB read between launches (outside the timed region), "
                    "each launch timed alone with events"}


def compare_dense(dev, peak, iters=20):
    """The 8B-shaped layer (batch 16, 32 q / 8 kv heads, 4096 tokens, pages of 128) on the
    same kernel and work line: 2-bit keys and values with 0 (KIVI), 16 and 32 (Kitty, 12.5%
    and 25%) boosted key channels, and the unquantized fp16 cache.  Decode attention only,
    each variant over replicas totalling at least 512 MB of cache."""
    import torch

    from bit_mixed_precision_channel_b200 import binding as kb
    from bit_mixed_precision_channel_b200 import synthetic as syn
    from bit_mixed_precision_channel_b200.cache import PagedKVCache

    w = syn.WORKLOADS[WORKLOAD]
    B, P, H, D, L = w.batch, w.P, w.Hkv, w.D, w.context
    n = L // P
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    sigma = torch.from_numpy(syn.key_channel_sigma(w)).to(dev)
    K = (torch_randn((B, L, H, D), gen, dev) * sigma).half()
    V = torch_randn((B, L, H, D), gen, dev).half()
    q = torch_randn((B, w.Hq, D), gen, dev).half()
    out = torch.empty(B, w.Hq, D, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def time_graph(fns, replicas):
        for f in fns:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in fns:
                f()
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(iters):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
        return a.elapsed_time(b) / iters / replicas

    res = {}
    for k in (0, 16, 32):
        cfg = kb.Config(head_dim=D, num_q_heads=w.Hq, num_kv_heads=H, page_tokens=P, key_group=w.G, num_boost=k,
                        dtype=w.dtype)
        payload = kb.page_layout(cfg)["payload_bytes"]
        reps = max(1, math.ceil(512e6 / (B * H * n * payload)))
        caches = [PagedKVCache(cfg, B, n + 1, B * (n + 1), device=dev) for _ in range(reps)]
        for c in caches:
            c.prefill_batch(K, V)
        ms = time_graph([(lambda c=c: c.attend(q, out)) for c in caches], reps)
        nbytes = B * H * n * payload + B * w.Hq * D * 6 + 4 * B * n + 8 * B
        res[f"2bit_k{k}"] = {"decode_us_per_launch": round(ms * 1e3, 2), "bytes_per_launch": nbytes,
                             "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "decode_tokens_per_s": round(B / (ms * 1e-3), 1),
                             "kv_bytes_per_token_head": round(payload / P, 2)}
        del caches
    cfg = kb.Config(head_dim=D, num_q_heads=w.Hq, num_kv_heads=H, page_tokens=P, key_group=w.G, num_boost=32,
                    dtype=w.dtype)
    page_bytes = B * H * n * kb.dense_page_bytes(cfg)
    reps = max(1, math.ceil(512e6 / page_bytes))
    table = torch.arange(B * n, dtype=torch.int32, device=dev).view(B, n)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    ws = torch.zeros(kb.decode_workspace_bytes(cfg, B, n), dtype=torch.uint8, device=dev)
    # [B][n][P][H][D] -> pages [B * n][H][2][P][D]
    pages = torch.stack([K.view(B, n, P, H, D), V.view(B, n, P, H, D)], dim=3)  # [B][n][P][2][H][D]
    pool = pages.permute(0, 1, 4, 3, 2, 5).contiguous().view(-1)
    pools = [pool] + [pool.clone() for _ in range(reps - 1)]
    ms = time_graph([(lambda p=p: kb.decode_attention_dense(cfg, p, q, table, lens, out, ws)) for p in pools], reps)
    nbytes = B * H * n * kb.dense_page_bytes(cfg) + B * w.Hq * D * 6 + 4 * B * n + 8 * B
    res["fp16_dense"] = {"decode_us_per_launch": round(ms * 1e3, 2), "bytes_per_launch": nbytes,
                         "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "decode_tokens_per_s": round(B / (ms * 1e-3), 1),
                         "kv_bytes_per_token_head": 512.0}
    dense_us = res["fp16_dense"]["decode_us_per_launch"]
    for key in ("2bit_k0", "2bit_k16", "2bit_k32"):
        res[key]["speedup_vs_fp16_dense"] = round(dense_us / res[key]["decode_us_per_launch"], 3)
        res[key]["kv_bytes_ratio_vs_fp16_dense"] = round(512.0 / res[key]["kv_bytes_per_token_head"], 2)
    res["what"] = ("one decode-attention launch per layer at batch 16, 4096-token prompts; the same kernel and "
                   "work line for every variant, the fp16 cache read through its page table in 16-token pieces")
    del pools, pool, pages, K, V
    torch.cuda.empty_cache()
    return res


def prefill_bench(dev, peak_tflops, L=4096, iters=10):
    """The MiniKV prefill path of one Llama-3-8B-shaped layer (32 q / 8 kv heads, one
    L-token prompt, fp16): prefill attention with cumulative scores, then 25% + 25%
    retention, gather and page quantization of the kept tokens.  The attention is bound
    by the tensor cores: its flops are the QK and PV products of the causal pass plus
    the QK products of the score pass."""
    import torch

    from bit_mixed_precision_channel_b200 import binding as kb
    from bit_mixed_precision_channel_b200 import synthetic as syn

    w = syn.WORKLOADS[WORKLOAD]
    Hq, H, D, P = w.Hq, w.Hkv, w.D, w.P
    cfg = kb.Config(head_dim=D, num_q_heads=Hq, num_kv_heads=H, page_tokens=P, key_group=w.G, num_boost=w.k,
                    dtype=w.dtype)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    sigma = torch.from_numpy(syn.key_channel_sigma(w)).to(dev)
    q = torch_randn((L, Hq, D), gen, dev).half()
    k = (torch_randn((L, H, D), gen, dev) * sigma).half()
    v = torch_randn((L, H, D), gen, dev).half()
    out = torch.empty(L, Hq, D, device=dev)
    scores = torch.empty(H, L, device=dev)
    ws = torch.zeros(kb.prefill_workspace_bytes(cfg, L), dtype=torch.uint8, device=dev)
    nh = nr = L // 4
    keep = torch.empty(H, L, dtype=torch.int32, device=dev)
    n_keep = torch.empty(H, dtype=torch.int32, device=dev)
    n = nh + nr
    k_out = torch.empty(n, H, D, dtype=torch.float16, device=dev)
    v_out = torch.empty_like(k_out)
    n_pages = n // P
    pool = torch.zeros(n_pages * H * kb.page_bytes(cfg), dtype=torch.uint8, device=dev)
    dst = torch.arange(n_pages, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def attn():
        kb.prefill_attention(cfg, q, k, v, out, scores, ws)

    def rest():
        kb.retain_tokens(cfg, scores, nh, nr, keep, n_keep)
        kb.gather_tokens(cfg, k, v, keep, n, k_out, v_out, err)
        kb.quantize_pages(cfg, kb.Source.token_major(k_out, cfg), kb.Source.token_major(v_out, cfg), dst, pool, err)

    def timeit(f):
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            f()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    ms_attn = timeit(attn)
    ms_rest = timeit(rest)
    assert int(err.item()) == 0
    pairs = L * (L + 1) / 2  # causal (query, key) pairs
    flops = Hq * pairs * D * 2 * 2 + Hq * pairs * D * 2  # forward QK + PV, score pass QK
    tf = flops / (ms_attn * 1e-3) / 1e12
    return {"tokens": L, "attention_ms": round(ms_attn, 4), "retain_gather_quantize_ms": round(ms_rest, 4),
            "tokens_per_s": round(L / ((ms_attn + ms_rest) * 1e-3), 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak_tflops, "unit": "TFLOP/s",
                         "frac": round(tf / peak_tflops, 4),
                         "peak_source": "measured bf16 cuBLAS (burst); fp16 has the same nominal rate"},
            "kept_tokens": n,
            "what": "one layer of one prompt: causal attention with cumulative scores (two passes), then "
                    "heavy-hitter + recent retention (25% + 25%), gather and quantization of the kept tokens"}


# ------------------------------------------------------------------ reference arm

def workload_config(w, layers, world, payload):
    """The bench's `config` object (both arms report the same one)."""
    B, P, D = w.batch, w.P, w.D
    n_pages = w.context // P
    return {"workload": f"Llama-3-8B-shaped decode: batch {B} per GPU, {w.Hq} q / {w.Hkv} kv heads, "
                        f"head_dim {D}, {w.context}-token prompts in pages of {P}, {w.k} of {D} key "
                        f"channels boosted to 4 bit, residual window {P}, {layers} layers per step",
            "global_batch": B * world, "layers": layers, "seq_len": w.context,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"inputs larger than L2: {layers} layer caches, "
                  f"{layers * B * w.Hkv * n_pages * payload / 1e9:.2f} GB of packed pages per GPU"}


def run_reference(args):
    """The oracle as the reference implementation: each step decodes a bounded sample
    (one sequence x kv-head unit per host thread, at least 8) of the same workload on the
    host cores."""
    import concurrent.futures as cf

    import oracle
    from bit_mixed_precision_channel_b200 import synthetic as syn

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    w = syn.WORKLOADS[WORKLOAD]
    oc = oracle.Cfg(D=w.D, Hq=w.Hq, Hkv=w.Hkv, P=w.P, G=w.G, k=w.k, dtype=w.dtype)
    P, D, g = w.P, w.D, w.gqa
    n_pages = w.context // P
    sigma = syn.key_channel_sigma(w)
    threads = max(1, min(os.cpu_count() or 1, 32))
    # at least one unit per thread, so that every host core has work
    units = [(b, h) for b in range(w.batch) for h in range(w.Hkv)][:max(threads, 8)]
    Ks = {b: syn.keys(w, b, 0, w.context, sigma) for b in {u[0] for u in units}}
    Vs = {b: syn.values(w, b, 0, w.context) for b in Ks}
    pools = {}
    for b in Ks:
        pool = np.zeros((n_pages, w.Hkv, oc.record_bytes), np.uint8)
        for i in range(n_pages):
            for h in range(w.Hkv):
                pool[i, h] = oracle.quantize_page(Ks[b][i * P:(i + 1) * P, h], Vs[b][i * P:(i + 1) * P, h], oc)
        pools[b] = pool
    kn, _ = syn.step_tokens(w, 0, sigma)
    q = syn.queries(w, 0)
    sm = 1.0 / math.sqrt(D)
    payload = oracle.layout(P, D, w.k, w.G)["payload_bytes"]
    res_len = 1

    def unit(bh):
        b, h = bh
        rk = kn[b, h][None]
        return oracle.decode_unit(pools[b], oc, h, list(range(n_pages)), rk, rk, q[b, h * g:(h + 1) * g], sm)

    per_unit = payload * n_pages + res_len * 2 * D * 2 + g * D * 6 + 4 * n_pages
    with cf.ThreadPoolExecutor(threads) as ex:
        for _ in range(args.warmup):
            list(ex.map(unit, units))
        t0 = time.perf_counter()
        for _ in range(args.steps):
            list(ex.map(unit, units))
        dt = time.perf_counter() - t0
    value = per_unit * len(units) * args.steps / dt / 1e9
    sample = (f"{len(units)} (sequence, kv head) decode units of one layer per step, fp64 attention over "
              f"{n_pages} pages + {res_len} residual token, {threads} threads")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.layers, args.gpus, payload),
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def decode_leg(name):
    """One full-size cache of a workload and five decode launches (for a profiler to
    capture the last ones); returns the workload's page bytes and launch count."""
    import torch

    from bit_mixed_precision_channel_b200 import binding as kb
    from bit_mixed_precision_channel_b200 import synthetic as syn
    from bit_mixed_precision_channel_b200.cache import PagedKVCache

    dev = torch.device("cuda")
    w = syn.WORKLOADS[name]
    cfg = kb.Config(head_dim=w.D, num_q_heads=w.Hq, num_kv_heads=w.Hkv, page_tokens=w.P, key_group=w.G,
                    num_boost=w.k, dtype=w.dtype)
    tdt = kb.torch_dtype(w.dtype)
    lens = syn.lengths(w)
    P = w.P
    pool_pages = int(sum(lens // P) + 2 * w.batch)
    sigma = torch.from_numpy(syn.key_channel_sigma(w)).to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    c = PagedKVCache(cfg, w.batch, int(max(lens) // P + 2), pool_pages, device=dev,
                     page_order=syn.page_order(w, pool_pages))
    for b, K, V in _device_prompts(w, lens, sigma, gen, tdt, dev):
        c.prefill(b, K, V)
    q = torch_randn((w.batch, w.Hq, w.D), gen, dev).to(tdt)
    out = torch.empty(w.batch, w.Hq, w.D, device=dev)
    for _ in range(5):
        c.attend(q, out)
    torch.cuda.synchronize()
    assert c.check_errors() == 0
    payload = kb.page_layout(cfg)["payload_bytes"]
    return {"leg": "decode", "workload": name, "page_bytes": int(sum(lens // P)) * w.Hkv * payload,
            "residual_tokens": int(sum(lens % P)), "launches": 5}


def main():
    args = parse()
    if args.leg == "minikv":
        import torch
        res = {"leg": "minikv", **prefill_bench(torch.device("cuda"), peak_tensor())}
    elif args.leg.startswith("decode:"):
        res = decode_leg(args.leg.split(":", 1)[1])
    else:
        res = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
