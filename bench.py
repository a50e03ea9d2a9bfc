#!/usr/bin/env python
"""Benchmark: GQA decode effective HBM GB/s on B200 (plus prefill TFLOP/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one token's attention work for a Llama-3-8B-shaped model: for each
of its 32 layers, the append of the new token's K/V rows and the decode of
the 8 x 32 query heads over the 8 x 8 KV heads at context 8192 (bf16, head
dim 128), as one gqa_decode_append call. Every layer has its own 256 MiB cache pair, so a step
streams 8 GiB, far more than the 126 MB L2; no flush is needed.

value = KV bytes that decode must read (each cached row once) / step time.
N > 1 runs independent replicas (one per GPU, no data-path collective): value
is the sum over ranks of the bytes processed divided by the slowest rank's
time.

--impl reference times the float64 CPU oracle on the host cores instead (the
reference arm), one (batch, KV head) unit of the same workload per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "llama3_8b_decode_b8_h32_k8_d128_s8192"
LAYERS = 32
METRIC = "GQA decode effective HBM GB/s"
UNIT = "GB/s"


# ---------------------------------------------------------------------------
# multi-rank plumbing (also exercised on CPU with gloo by the tests)

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def aggregate(local_ms: float, local_bytes: float, group=None):
    """(max time over ranks in ms, total bytes over ranks) via all_reduce."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return local_ms, local_bytes
    backend = dist.get_backend(group)
    dev = "cuda" if backend == "nccl" else "cpu"
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    b = torch.tensor([local_bytes], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(b, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), float(b.item())


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML polling thread)

class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, interval_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.index, self.interval = index, interval_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self._nv, self.error = None, str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self._nv:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self._nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        reasons = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": reasons}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def profiled_traffic(name: str, source_files):
    """ncu DRAM bytes per launch from profiles/<name>.json, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", f"{name}.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    h = hashlib.sha256()
    for s in source_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    if rec.get("source_sha256") != h.hexdigest():
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# our arm

def bench_ours(args, rank, world, local):
    import torch

    from kv_cache_02_b200 import gqa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.DECODE_WORKLOADS[WORKLOAD]
    inp = synth.decode_inputs(w)
    B, H, K, d, S = w.B, w.H, w.K, w.d, w.S_max
    scale = 1.0 / np.sqrt(d)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).to(dev)

    kc1, vc1 = to_dev(inp["k_cache"]), to_dev(inp["v_cache"])
    kc = torch.empty((LAYERS, B, K, S, d), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    for layer in range(LAYERS):
        kc[layer].copy_(kc1)
        vc[layer].copy_(vc1)
    del kc1, vc1
    q = to_dev(inp["q"]).unsqueeze(0).repeat(LAYERS, 1, 1, 1).contiguous()
    k_new = to_dev(inp["k_new"]).unsqueeze(0).repeat(LAYERS, 1, 1, 1).contiguous()
    v_new = to_dev(inp["v_new"]).unsqueeze(0).repeat(LAYERS, 1, 1, 1).contiguous()
    pos = to_dev(inp["pos"])
    seqlens = to_dev(inp["seqlens"])
    out = torch.empty_like(q)
    ws_bytes = gqa.gqa_decode_workspace_bytes(B, H, K, S, d, 0)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    launches_per_layer = 2 if ws_bytes > 16 else 1  # decode with the append, + the combine when split
    kv_bytes_layer = 2 * B * K * S * d * 2  # K and V, every row once
    stream = torch.cuda.current_stream()

    layer_args = [(out[layer], q[layer], kc[layer], vc[layer], k_new[layer], v_new[layer]) for layer in range(LAYERS)]

    def step():
        for o, qq, k, v, kn, vn in layer_args:
            # the new token's K/V go into the cache at row pos, then every head
            # attends over pos + 1 keys: one fused pass per layer
            gqa.gqa_decode_append(o, qq, k, v, kn, vn, pos, scale, 0, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = gqa.gqa_get_last_error()
    if status != (0, 0):
        raise RuntimeError(f"device error during warm-up: {status}")

    # the step as a CUDA graph: the same 32 calls, captured once and replayed,
    # so no launch waits on the host. Thread-local capture: other threads of
    # the process (a process group's watchdog) may keep using CUDA meanwhile.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    import torch.distributed as dist

    def timed(run, steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(steps):
            run()
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return t0.elapsed_time(t1)

    with ClockSampler(local) as clocks:
        local_ms = timed(graph.replay, args.steps)
    status = gqa.gqa_get_last_error()
    if status != (0, 0):
        raise RuntimeError(f"device error in the timed region: {status}")
    max_ms, total_bytes = aggregate(local_ms, kv_bytes_layer * LAYERS * args.steps)
    value = total_bytes / (max_ms * 1e-3) / 1e9
    ms_per_step = max_ms / args.steps

    # the same step with the 32 calls issued one by one from Python
    eager_steps = max(3, min(args.steps, 50))
    eager_ms, eager_bytes = aggregate(timed(step, eager_steps), kv_bytes_layer * LAYERS * eager_steps)
    del graph

    # end to end through the public API: every step copies its inputs in from
    # pinned host memory and its output back out. The copies run on a second
    # stream over two buffer sets, so step s+1's inputs arrive and step s-1's
    # output leaves while step s computes; the timed region ends when the last
    # output is on the host.
    q_h = q.cpu().pin_memory()
    kn_h, vn_h = k_new.cpu().pin_memory(), v_new.cpu().pin_memory()
    pos_h = pos.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    sets = [(q, k_new, v_new, pos, out),
            (torch.empty_like(q), torch.empty_like(k_new), torch.empty_like(v_new), torch.empty_like(pos),
             torch.empty_like(out))]
    copy_stream = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in sets]    # inputs of the set copied in
    ev_done = [torch.cuda.Event() for _ in sets]  # the set's step computed
    ev_out = torch.cuda.Event()                   # last output copied out

    def copy_in(i):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_done[i])  # the step that last used the set is finished
            for dst, src in zip(sets[i][:4], (q_h, kn_h, vn_h, pos_h)):
                dst.copy_(src, non_blocking=True)
            ev_in[i].record(copy_stream)

    def compute(i):
        stream.wait_event(ev_in[i])
        qq, kn, vn, ps, oo = sets[i]
        for layer in range(LAYERS):
            gqa.gqa_decode_append(oo[layer], qq[layer], kc[layer], vc[layer], kn[layer], vn[layer], ps, scale, 0, ws)
        ev_done[i].record(stream)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_done[i])
            out_h.copy_(oo, non_blocking=True)
            ev_out.record(copy_stream)

    def e2e_run(steps):
        copy_in(0)
        for s_ in range(steps):
            if s_ + 1 < steps:
                copy_in((s_ + 1) % 2)
            compute(s_ % 2)
        stream.wait_event(ev_out)

    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms_local = e0.elapsed_time(e1)
    e2e_max_ms, e2e_bytes = aggregate(e2e_ms_local, kv_bytes_layer * LAYERS * e2e_steps)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, kn_h, vn_h, pos_h))
    d2h = out_h.numel() * out_h.element_size()
    status = gqa.gqa_get_last_error()
    if status != (0, 0):
        raise RuntimeError(f"device error in the end-to-end run: {status}")

    peaks, peak_src = measured_peaks()
    # every launch in the timed region is this call (decode kernel + combine):
    # its average duration is the region over the calls, gaps included
    dec_avg_ms = max_ms / (args.steps * LAYERS)
    achieved = kv_bytes_layer / (dec_avg_ms * 1e-3) / 1e9
    traffic = profiled_traffic("decode_bf16_llama3_8b_traffic",
                               ["kv_cache_02_b200/csrc/decode.cuh", "kv_cache_02_b200/csrc/common.cuh"])
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "H": H, "K": K, "d": d, "context": S,
                   "layers_per_step": LAYERS, "kv_append_per_layer": "fused into the decode pass",
                   "step": "the 32 gqa_decode_append calls captured once as a CUDA graph and replayed",
                   "l2": "inputs larger than L2: each step streams 32 distinct 256 MiB cache pairs (8 GiB)",
                   "parallelism": f"replicas x{world}", "num_splits": "auto"},
        "roofline": {"bound": "hbm", "kernel": "gqa_decode_append (decode_bf16_kernel with the append + decode_combine_kernel)",
                     "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "peak_source": peak_src,
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": traffic, "algorithmic_bytes_per_launch": kv_bytes_layer,
                     "avg_launch_ms": round(dec_avg_ms, 5),
                     "avg_launch_from": "timed region / calls (every launch in it is this call)"},
        "eager": {"value": round(eager_bytes / (eager_ms * 1e-3) / 1e9, 1), "unit": UNIT, "steps": eager_steps,
                  "note": "the same step with the calls issued one by one from Python"},
        "e2e": {"value": round(e2e_bytes / (e2e_max_ms * 1e-3) / 1e9, 1), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "pinned-host q, k_new, v_new, pos copied in and out copied back every step, on a "
                        "second stream over two buffer sets (overlapping the neighbouring steps' compute); "
                        "the calls issued one by one from Python; the KV cache is device-resident state"},
        "gpu_launches": launches_per_layer * LAYERS * args.steps,
        "clocks": clocks.summary(),
    }
    return result, dict(inp=inp, scale=scale, kv_bytes_layer=kv_bytes_layer)


DECODE_EXTRA = ["ragged_70b_decode_b32_h64_k8_d128_s1k_16k", "long_ctx_gqa_b1_h64_k8_d128_s131072",
                "long_ctx_mqa_b1_h64_k1_d128_s131072"]
PREFILL = "causal_prefill_b4_s4096_h32_k8_d128"
PAGED_EXTRA = list(synth.PAGED_WORKLOADS)
INT8_EXTRA = list(synth.INT8_WORKLOADS)
VARLEN_EXTRA = list(synth.VARLEN_WORKLOADS)
PROJ_EXTRA = list(synth.PROJ_WORKLOADS)


class L2Flush:
    """Evict L2 between timed iterations: write a buffer 4x larger than L2, then
    read another one, so that L2 is left holding clean lines (a write alone
    would leave ~126 MB of dirty lines whose write-back the next kernel pays)."""

    def __init__(self, nbytes: int = 512 * 1024 * 1024):
        import torch

        self.w = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(nbytes // 4, dtype=torch.int32, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.max()


def back_to_back_ms(make_call, nbytes: int, reps: int) -> float:
    """Per-call ms of calls run back to back from a CUDA graph. make_call(i)
    builds a call over input copy i; the graph cycles through enough copies
    that together they hold at least twice the L2 size of distinct rows, so
    no call finds the rows it reads in L2 (the inputs are larger than L2)."""
    import torch

    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    copies = min(16, max(1, -(-2 * l2 // max(nbytes, 1))))
    calls = [make_call(i) for i in range(copies)]
    n = copies * max(1, -(-16 // copies))  # at least 16 calls per replay
    for c in calls:  # eager once: one-time setup outside the capture
        c()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        for i in range(n):
            calls[i % copies]()
    graph.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / n)
    del graph, calls
    return statistics.median(times)


BACK_TO_BACK = "calls back to back from a CUDA graph over rotating input copies (>= 2x L2 of distinct rows)"


def isolated_ms(make_call, reps: int, n: int = 16) -> float:
    """Per-call ms of calls that each follow an L2 flush, so that no call
    overlaps another or finds its rows in L2: a CUDA graph of n (flush, call)
    pairs less a graph of n flushes alone, over n."""
    import torch

    flush = L2Flush()
    call = make_call(0)
    call()
    torch.cuda.synchronize()
    graphs = []
    for with_call in (True, False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for _ in range(n):
                flush()
                if with_call:
                    call()
        graphs.append(g)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    diffs = []
    for _ in range(reps):
        t = []
        for g in graphs:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            t.append(a.elapsed_time(b))
        diffs.append((t[0] - t[1]) / n)
    del graphs, flush
    return statistics.median(diffs)


ISOLATED = "each call after an L2 flush (a graph of flush + call pairs less a graph of flushes, per call)"

KV_APPEND = "kv_append_b8_k8_d128_s8192"
PROMPT_WRITE = "prompt_cache_write_b4_s4096_k8_d128"
MEANPOOL = "meanpool_kv_h64_k8_d128_dm8192"
SMALL_EXTRA = [KV_APPEND, PROMPT_WRITE, MEANPOOL]


def small_kernel_measurements(args, peaks, steps, only=None):
    """The HBM-bound kernels beside the decode: the append of one token (latency), the prompt's
    K/V written to the cache (the bulk form of the append), and mean pooling of K/V projection
    weights from 64 heads to 8."""
    import torch

    from kv_cache_02_b200 import gqa

    res = {}
    if only in (None, KV_APPEND):
        # gqa_kv_append at the Llama-3-8B decode layer's shape: 2 B K rows of 256 bytes
        B, K, d, S_max = 8, 8, 128, 8192
        kn = torch.randn((B, K, d), device="cuda").to(torch.bfloat16)
        vn = torch.randn((B, K, d), device="cuda").to(torch.bfloat16)
        pos = torch.full((B,), S_max - 1, dtype=torch.int32, device="cuda")

        def make_call(i):
            kc = torch.empty((B, K, S_max, d), dtype=torch.bfloat16, device="cuda")
            vc = torch.empty_like(kc)
            return lambda: gqa.gqa_kv_append(kc, vc, kn, vn, pos)

        ms = back_to_back_ms(make_call, 256 << 20, steps)
        byts = 2 * 2 * B * K * d * 2  # the new rows read, and written into the caches
        res[KV_APPEND] = {"ms": round(ms, 5), "bytes": byts, "GB/s": round(byts / (ms * 1e-3) / 1e9, 1),
                          "bound": "launch latency (64 KiB moved)", "timing": "calls back to back from a CUDA graph"}
        del kn, vn, pos
    if only in (None, PROMPT_WRITE):
        # the prompt's K/V [B,S,K,d] into the caches [B,K,S_max,d]: the causal prefill with the cache
        # write less the prefill without it, each after an L2 flush
        w = synth.PREFILL_WORKLOADS[PREFILL]
        q = torch.randn((w.B, w.S, w.H, w.d), device="cuda").to(torch.bfloat16)
        k = torch.randn((w.B, w.S, w.K, w.d), device="cuda").to(torch.bfloat16)
        v = torch.randn_like(k)
        out = torch.empty_like(q)
        kc = torch.empty((w.B, w.K, w.S, w.d), dtype=torch.bfloat16, device="cuda")
        vc = torch.empty_like(kc)
        flush = L2Flush()
        t = {True: [], False: []}
        for it in range(args.warmup + steps):
            for with_cache in (True, False):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                if with_cache:
                    gqa.gqa_prefill_causal(out, q, k, v, 1.0 / np.sqrt(w.d), kc, vc)
                else:
                    gqa.gqa_prefill_causal(out, q, k, v, 1.0 / np.sqrt(w.d))
                b.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    t[with_cache].append(a.elapsed_time(b))
        ms = statistics.median(t[True]) - statistics.median(t[False])
        byts = w.B * w.S * w.K * w.d * 2 * 2  # the K and V rows written to the caches
        res[PROMPT_WRITE] = {"increment_ms": round(ms, 5), "bytes_written": byts,
                             "with_write_ms": round(statistics.median(t[True]), 5),
                             "without_write_ms": round(statistics.median(t[False]), 5),
                             "how": "the prefill stores each key tile to the cache from shared memory while it "
                                    "computes (no separate pass); the increment is what the stores cost it",
                             "timing": "gqa_prefill_causal with the cache write less without it, medians, "
                                       "each call after an L2 flush"}
        del q, k, v, out, kc, vc, flush
    if only in (None, MEANPOOL):
        # W_K of 64 heads [64, 128, 8192] -> 8 KV heads: 128 MiB read, 16 MiB written
        H, K, d, dm = 64, 8, 128, 8192
        dst = torch.empty((1, K, d * dm), dtype=torch.bfloat16, device="cuda")

        def make_call(i):
            src = torch.randn((1, H, d * dm), device="cuda").to(torch.bfloat16)
            return lambda: gqa.gqa_meanpool_kv(dst, src)

        src_bytes = H * d * dm * 2
        ms = back_to_back_ms(make_call, src_bytes, steps)
        byts = src_bytes + K * d * dm * 2
        gbs = byts / (ms * 1e-3) / 1e9
        res[MEANPOOL] = {"ms": round(ms, 5), "bytes": byts, "GB/s": round(gbs, 1),
                         "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4), "timing": BACK_TO_BACK}
        del dst
    if gqa.gqa_get_last_error() != (0, 0):
        raise RuntimeError("device error in the small-kernel measurements")
    torch.cuda.empty_cache()
    return res


def extra_measurements(args, only=None):
    """Other workloads, rank 0 at N = 1: decode configs and the causal prefill."""
    import torch

    from kv_cache_02_b200 import gqa

    peaks, _ = measured_peaks()
    res = {}
    for name in DECODE_EXTRA:
        if only is not None and name != only:
            continue
        w = synth.DECODE_WORKLOADS[name]
        inp = synth.decode_inputs(w)

        def to_dev(a):
            t = torch.from_numpy(np.ascontiguousarray(a))
            return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).cuda()

        q, lens = to_dev(inp["q"]), to_dev(inp["seqlens"])
        out = torch.empty_like(q)
        wsb = gqa.gqa_decode_workspace_bytes(w.B, w.H, w.K, w.S_max, w.d, 0)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
        kv_bytes = int(inp["seqlens"].astype(np.int64).sum()) * w.K * w.d * 2 * 2

        def make_call(i):
            kc, vc = to_dev(inp["k_cache"]), to_dev(inp["v_cache"])
            return lambda: gqa.gqa_decode(out, q, kc, vc, lens, 1.0 / np.sqrt(w.d), 0, ws)

        ms = back_to_back_ms(make_call, kv_bytes, args.steps if only else 20)
        if gqa.gqa_get_last_error() != (0, 0):
            raise RuntimeError(f"device error in {name}")
        gbs = kv_bytes / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 5), "kv_bytes": kv_bytes, "GB/s": round(gbs, 1),
                     "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4), "timing": BACK_TO_BACK}
        if kv_bytes < 256 << 20:  # a short call: also timed on its own
            ims = isolated_ms(make_call, args.steps if only else 10)
            igbs = kv_bytes / (ims * 1e-3) / 1e9
            res[name]["isolated"] = {"ms": round(ims, 5), "GB/s": round(igbs, 1),
                                     "frac_of_measured_hbm": round(igbs / peaks["hbm_gbs"], 4), "timing": ISOLATED}
        del q, out, ws
        torch.cuda.empty_cache()
    # paged caches: the same workloads' values over randomly placed blocks
    for name in PAGED_EXTRA:
        if only is not None and name != only:
            continue
        res[name] = paged_measurement(args, name, peaks, 20 if only is None else args.steps)
    for name in INT8_EXTRA:
        if only is not None and name != only:
            continue
        res[name] = int8_measurement(args, name, peaks, 20 if only is None else args.steps)
    for name in VARLEN_EXTRA:
        if only is not None and name != only:
            continue
        res[name] = varlen_measurement(args, name, peaks, 20 if only is None else args.steps)
    for name in PROJ_EXTRA:
        if only is not None and name != only:
            continue
        res[name] = proj_measurement(args, name, peaks, 20 if only is None else args.steps)
    if only is None or only in SMALL_EXTRA:
        res.update(small_kernel_measurements(args, peaks, 20 if only is None else args.steps, only))
    if only is not None and only != PREFILL:
        return res
    # causal prefill with the KV-cache write: FLOPs over the causal pairs (j <= i) only
    w = synth.PREFILL_WORKLOADS[PREFILL]
    inp = synth.prefill_inputs(w)

    def to_dev2(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()

    q, k, v = to_dev2(inp["q"]), to_dev2(inp["k"]), to_dev2(inp["v"])
    out = torch.empty_like(q)
    kc = torch.empty((w.B, w.K, w.S, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    flops = 4.0 * w.B * w.H * w.d * w.S * (w.S + 1) / 2
    times = []
    flush = L2Flush()
    for it in range(args.warmup + (args.steps if only else 20)):
        flush()  # no K/V tile of the previous call left in L2
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        gqa.gqa_prefill_causal(out, q, k, v, 1.0 / np.sqrt(w.d), kc, vc)
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    tf = flops / (ms * 1e-3) / 1e12
    res[w.name] = {"ms": round(ms, 4), "flops": flops, "TFLOP/s": round(tf, 1),
                   "frac_of_measured_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                   "frac_of_measured_bf16_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                   "includes": "attention + KV-cache write", "l2": "flushed (512 MiB write, then 512 MiB read)"}
    del flush
    if gqa.gqa_get_last_error() != (0, 0):
        raise RuntimeError("device error in extra measurements")
    return res


def paged_measurement(args, name, peaks, steps):
    """gqa_decode_paged (gqa_decode_append_paged for a workload with an append) of one paged workload."""
    import torch

    from kv_cache_02_b200 import gqa

    pw = synth.PAGED_WORKLOADS[name]
    w = synth.DECODE_WORKLOADS[pw.base]
    inp = synth.paged_inputs(pw)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).cuda()

    q, table = to_dev(inp["q"]), to_dev(inp["block_table"])
    out = torch.empty_like(q)
    wsb = gqa.gqa_decode_paged_workspace_bytes(w.B, w.H, w.K, w.d, pw.block_size, table.shape[1], 0)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(w.d)
    if w.append:
        pos, kn, vn = to_dev(inp["pos"]), to_dev(inp["k_new"]), to_dev(inp["v_new"])
        lens = inp["pos"].astype(np.int64) + 1

        def make_call(i):
            kp, vp = to_dev(inp["k_pool"]), to_dev(inp["v_pool"])
            return lambda: gqa.gqa_decode_append_paged(out, q, kp, vp, kn, vn, table, pos, scale, 0, ws)
    else:
        sl = to_dev(inp["seqlens"])
        lens = inp["seqlens"].astype(np.int64)

        def make_call(i):
            kp, vp = to_dev(inp["k_pool"]), to_dev(inp["v_pool"])
            return lambda: gqa.gqa_decode_paged(out, q, kp, vp, table, sl, scale, 0, ws)
    kv_bytes = int(lens.sum()) * w.K * w.d * 2 * 2
    ms = back_to_back_ms(make_call, kv_bytes, steps)
    if gqa.gqa_get_last_error() != (0, 0):
        raise RuntimeError(f"device error in {name}")
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    r = {"ms": round(ms, 5), "kv_bytes": kv_bytes, "GB/s": round(gbs, 1),
         "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4), "block_size": pw.block_size,
         "call": "gqa_decode_append_paged" if w.append else "gqa_decode_paged", "timing": BACK_TO_BACK}
    del q, table, out, ws
    torch.cuda.empty_cache()
    return r


def int8_measurement(args, name, peaks, steps):
    """gqa_decode_int8 over an 8-bit cache: bytes = the codes and scales of every valid row."""
    import torch

    from kv_cache_02_b200 import gqa

    inp = synth.int8_inputs(name)
    B, H, d = inp["q"].shape
    K, S_max = inp["k_codes"].shape[1:3]

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).cuda()

    q, sl = to_dev(inp["q"]), to_dev(inp["seqlens"])
    out = torch.empty_like(q)
    wsb = gqa.gqa_decode_int8_workspace_bytes(B, H, K, S_max, d, 0)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    kv_bytes = int(inp["seqlens"].astype(np.int64).sum()) * K * (d + 4) * 2

    def make_call(i):
        kc, ks, vc, vs = (to_dev(inp[k]) for k in ("k_codes", "k_scale", "v_codes", "v_scale"))
        return lambda: gqa.gqa_decode_int8(out, q, kc, ks, vc, vs, sl, 1.0 / np.sqrt(d), 0, ws)

    ms = back_to_back_ms(make_call, kv_bytes, steps)
    if gqa.gqa_get_last_error() != (0, 0):
        raise RuntimeError(f"device error in {name}")
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    r = {"ms": round(ms, 5), "kv_bytes": kv_bytes, "GB/s": round(gbs, 1),
         "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4), "call": "gqa_decode_int8",
         "bytes": "int8 codes + one float scale per row", "timing": BACK_TO_BACK}
    del q, out, ws
    torch.cuda.empty_cache()
    return r


def varlen_measurement(args, name, peaks, steps):
    """gqa_prefill_causal_varlen (with the cache write): FLOPs over every sequence's causal pairs."""
    import torch

    from kv_cache_02_b200 import gqa

    w = synth.VARLEN_WORKLOADS[name]
    inp = synth.varlen_inputs(w)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).cuda()

    q, k, v, cu = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), to_dev(inp["cu_seqlens"])
    out = torch.empty_like(q)
    kc = torch.empty((w.B, w.K, w.S_max, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    lens = inp["lens"].astype(np.float64)
    flops = float(np.sum(4.0 * w.H * w.d * lens * (lens + 1) / 2))
    times = []
    flush = L2Flush()
    for it in range(args.warmup + steps):
        flush()  # no K/V tile of the previous call left in L2
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        gqa.gqa_prefill_causal_varlen(out, q, k, v, cu, 1.0 / np.sqrt(w.d), kc, vc)
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            times.append(a.elapsed_time(b))
    if gqa.gqa_get_last_error() != (0, 0):
        raise RuntimeError(f"device error in {name}")
    ms = statistics.median(times)
    tf = flops / (ms * 1e-3) / 1e12
    r = {"ms": round(ms, 4), "flops": flops, "TFLOP/s": round(tf, 1), "tokens": int(lens.sum()),
         "frac_of_measured_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
         "includes": "attention + KV-cache write", "l2": "flushed (512 MiB write, then 512 MiB read)"}
    del q, k, v, cu, out, kc, vc, flush
    torch.cuda.empty_cache()
    return r


def proj_measurement(args, name, peaks, steps):
    """gqa_kv_project_append: a decode step is bound by streaming W_KV (GB/s of weights and activations),
    a prompt by the tensor cores (TFLOP/s)."""
    import torch

    from kv_cache_02_b200 import gqa

    w = synth.PROJ_WORKLOADS[name]
    inp = synth.proj_inputs(w)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).cuda()

    x, wk, pos = to_dev(inp["x"]), to_dev(inp["w_kv"]), to_dev(inp["pos"])
    kc = torch.zeros((w.B, w.K, w.S_max, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    wsb = gqa.gqa_kv_project_workspace_bytes(w.B, w.T, w.K, w.d, w.d_model)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    M, N = w.B * w.T, w.K * 2 * w.d
    flops = 2.0 * M * N * w.d_model
    byts = (N * w.d_model + M * w.d_model + M * N) * 2  # W, x read once; the K/V rows written
    if M < 512:
        # a decode step's projection, HBM-bound and a few microseconds long: timed like the decode
        # workloads, back to back from a CUDA graph over rotating W_KV copies (>= 2x L2 of distinct
        # weights), as the calls of a model's layers run; and each call alone after an L2 flush
        def make_call(i):
            wi = wk if i == 0 else to_dev(inp["w_kv"])
            return lambda: gqa.gqa_kv_project_append(kc, vc, x, wi, pos, ws)

        ms = back_to_back_ms(make_call, N * w.d_model * 2, steps)
        ims = isolated_ms(make_call, steps)
        if gqa.gqa_get_last_error() != (0, 0):
            raise RuntimeError(f"device error in {name}")
        gbs, igbs = byts / (ms * 1e-3) / 1e9, byts / (ims * 1e-3) / 1e9
        r = {"ms": round(ms, 5), "flops": flops, "bytes": byts, "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1),
             "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4), "timing": BACK_TO_BACK,
             "isolated": {"ms": round(ims, 5), "GB/s": round(igbs, 1),
                          "frac_of_measured_hbm": round(igbs / peaks["hbm_gbs"], 4), "timing": ISOLATED}}
        del x, wk, pos, kc, vc, ws
        torch.cuda.empty_cache()
        return r
    flush = L2Flush()
    times = []
    for it in range(args.warmup + steps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        gqa.gqa_kv_project_append(kc, vc, x, wk, pos, ws)
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            times.append(a.elapsed_time(b))
    if gqa.gqa_get_last_error() != (0, 0):
        raise RuntimeError(f"device error in {name}")
    ms = statistics.median(times)
    r = {"ms": round(ms, 5), "flops": flops, "bytes": byts, "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1),
         "GB/s": round(byts / (ms * 1e-3) / 1e9, 1), "l2": "flushed (512 MiB write, then 512 MiB read)",
         "frac_of_measured_bf16_burst": round(flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    del x, wk, pos, kc, vc, ws, flush
    torch.cuda.empty_cache()
    return r


def cpu_baseline(inp, scale, kv_bytes_layer):
    """The oracle as it stands, on all host cores, over one full layer of the workload."""
    import oracle

    threads = synth.host_threads()
    # passes over one layer until about 10 s of host work (a bounded sample of the step)
    passes, t = 0, time.perf_counter()
    while True:
        oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale, nthreads=threads)
        passes += 1
        dt = time.perf_counter() - t
        if dt >= 10.0 or passes >= 1000:
            break
    return {"value": round(passes * kv_bytes_layer / dt / 1e9, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{passes} passes over one layer of the step (all 8 x 32 heads over 8192 keys), {dt:.1f} s"}


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores

def bench_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle

    w = synth.DECODE_WORKLOADS[WORKLOAD]
    inp = synth.decode_inputs(w)
    threads = synth.host_threads()
    scale = 1.0 / np.sqrt(w.d)
    # one (batch, KV head) unit per step: all G query heads of that group over the full context
    sel_all = [np.array([[b, g * w.G + j] for j in range(w.G)], np.int32) for b in range(w.B) for g in range(w.K)]
    unit_bytes = 2 * w.S_max * w.d * 2
    for i in range(args.warmup):
        oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale, sel=sel_all[i % len(sel_all)],
                      nthreads=threads)
    t = time.perf_counter()
    for i in range(args.steps):
        oracle.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"], scale, sel=sel_all[i % len(sel_all)],
                      nthreads=threads)
    dt = time.perf_counter() - t
    value = unit_bytes * args.steps / dt / 1e9
    sample = "one (batch, KV head) unit per step: 4 query heads over 8192 keys"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "K": w.K, "d": w.d, "context": w.S_max,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads and the CPU baseline")
    ap.add_argument("--only", choices=DECODE_EXTRA + PAGED_EXTRA + INT8_EXTRA + VARLEN_EXTRA + PROJ_EXTRA + SMALL_EXTRA
                    + [PREFILL],
                    default=None,
                    help="time one other workload alone (for profiling); prints its own JSON, not the contract line")
    ap.add_argument("--layers", type=int, default=32,
                    help="layers per step (32 for the model; fewer only for small profiling captures)")
    args = ap.parse_args()
    global LAYERS
    LAYERS = args.layers
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_env()

    if args.only:
        print(json.dumps({"only": args.only, **extra_measurements(args, args.only)}), flush=True)
        return

    if args.impl == "reference":
        res = bench_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        res, ctx = bench_ours(args, rank, world, local)
        if rank == 0:
            if world == 1 and not args.no_extra:
                res["cpu_baseline"] = cpu_baseline(ctx["inp"], ctx["scale"], ctx["kv_bytes_layer"])
                res["extra"] = extra_measurements(args)
            elif world == 1:
                res["cpu_baseline"] = None
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
