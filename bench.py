#!/usr/bin/env python
"""Benchmark: paged 8-bit-KV attention on B200.

One step = one decode step of the batch-8 workload (8 sequences x 32,768
cached tokens, 32 query / 4 KV heads, head_dim 128, block 16, FP8 E4M3 cache
with per-KV-head scales, 1% outlier channels x8): write + quantize the step's
new token into the paged cache and attend over the whole cache, in one call
(pkvq_paged_attn_decode_append: the split kernel writes the new tokens of its
blocks first, then the merge kernel).  The metric
is KV-read GB/s: the K and V code bytes one step must read (268,435,456 B per
GPU) divided by the step time.

The other four named workloads are measured in the same run under
"secondary", each against its own roofline and beside the FP64 oracle timed
on the host cores: the 1 x 1K decode (latency), the 8K causal prefill and the
8K chunk over a 120K prefix (useful TFLOP/s against the measured dense fp16 /
bf16 tensor peak), the 2 x 512K + 4 x 256K INT8 verify decode (KV GB/s
against HBM), and the KV writes of the two prefills.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pkvq|reference]
    python bench.py --only decode|prefill|kv_write [--workload n] [--steps K] [--warmup W]

--only runs nothing but W + K calls of one kernel path on its workload and
prints their average time: the command the ncu captures are taken with.

Under torchrun every rank runs the same batch on its own GPU (no collective on
the data path: weak scaling); the time is the max over ranks.  The reference
arm (--impl reference) times the FP64 CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DECODE_WORKLOAD = 2
METRIC = "paged FP8-KV attention: decode KV-read GB/s"


def decode_config(spec, world: int):
    return {"workload": spec.name, "batch": 8, "context": 32768, "q_heads": 32,
            "kv_heads": 4, "head_dim": 128, "block_size": 16, "kv_dtype": "fp8_e4m3",
            "step": "paged_attn_decode_append: new token's KV write + decode in one call",
            "l2": "inputs larger than L2: two 268 MB caches alternated step by step",
            "parallelism": f"dp{world} (independent batches per GPU)"}
PREFILL_WORKLOAD = 3
REFERENCE_BUDGET_S = 120.0
E2E_GRAPH_STEPS = 8
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
MIN_TIMED_S = 0.2          # every per-kernel number: at least this much replay time


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["pkvq", "reference"], default="pkvq")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip every secondary workload")
    ap.add_argument("--only", choices=["decode", "prefill", "kv_write"], default=None)
    ap.add_argument("--workload", type=int, default=None,
                    help="with --only: the named workload to run (decode 1, 2, 5; prefill "
                         "and kv_write 3, 4)")
    ap.add_argument("--ctx-div", type=int, default=1,
                    help="with --only decode: divide every context length by this (a smaller "
                         "case of the same shape, e.g. for a profiler capture)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(
            d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        self.active = threading.Event()   # samples are taken only while set
        self.active.set()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()
        self._t = None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if r & bit and bit != 0x1:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            if self.active.is_set():
                self._sample()
            time.sleep(self.period)

    def pause(self):
        self.active.clear()

    def resume(self):
        self.active.set()

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ CPU oracle --

def _bits16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_cache(case, only_seqs=None):
    """The oracle's own copy of the case's cache (quantized by the oracle);
    only_seqs: write just those sequences' tokens (a bounded sample)."""
    import oracle
    s = case.spec
    oc = oracle.Cache(s.kv_dtype, case.num_blocks, s.block_size, s.num_kv_heads, s.head_dim,
                      None if case.k_scale is None else case.k_scale.numpy(),
                      None if case.v_scale is None else case.v_scale.numpy(),
                      scale_per_layer=s.scale_per_layer)
    if only_seqs is None:
        oc.write(_bits16(case.k), _bits16(case.v), case.slot_mapping.numpy())
    else:
        for b in only_seqs:
            lo, hi = int(case.token_offsets[b]), int(case.token_offsets[b + 1])
            oc.write(_bits16(case.k[lo:hi]), _bits16(case.v[lo:hi]),
                     case.slot_mapping[lo:hi].numpy())
    return oc


def _oracle_rows(oc, case, rows, nthreads=0):
    """One oracle pass over the given (query token, head) rows; seconds, threads."""
    import oracle
    t0 = time.perf_counter()
    _, _, used = oracle.paged_attention(oc, _bits16(case.q), case.cu_seqlens_q.numpy(),
                                        case.context_lens.numpy(), case.block_table.numpy(),
                                        case.softmax_scale,
                                        rows=np.asarray(rows, np.int32).reshape(-1, 2),
                                        nthreads=nthreads)
    return time.perf_counter() - t0, used


def _row_bytes(spec) -> float:
    """Algorithmic KV bytes per (sequence, query head) row of a q_len-1 decode
    with equal lengths: a 1/Hq share of its sequence's KV bytes (the G rows
    of a KV head read the same codes)."""
    return synth.kv_read_bytes(spec) / len(spec.context_lens) / spec.num_q_heads


def _row_work(case, rows, unit: str) -> float:
    """Algorithmic work of the given (query token, head) rows: their share of
    the KV bytes (decode: a row reads 1 / (Hq * q_len) of its sequence's
    bytes) or their useful flops (4 * D per visible key)."""
    s = case.spec
    cu = case.cu_seqlens_q.numpy()
    seq = np.searchsorted(cu, np.asarray(rows)[:, 0], side="right") - 1
    tot = 0.0
    per_tok = synth.kv_read_bytes(synth.CaseSpec(s.kind, s.kv_dtype, s.num_q_heads,
                                                 s.num_kv_heads, [1], [1]))
    for (i, _), b in zip(rows, seq):
        c, ql = s.context_lens[b], s.q_lens[b]
        if unit == "GB/s":
            tot += c * per_tok / (s.num_q_heads * ql)
        else:
            tot += 4 * s.head_dim * max(0, c - ql + (i - cu[b]) + 1)
    return tot


def oracle_rate(case, oc, rows, unit: str, nthreads: int = 0, min_seconds: float = 3.0,
                max_passes: int = 50):
    """The FP64 oracle on `rows`, repeated until about min_seconds: returns
    (value in `unit`, seconds, threads, passes)."""
    total, passes, used = 0.0, 0, 0
    while passes < max_passes and (passes == 0 or total < min_seconds):
        dt, used = _oracle_rows(oc, case, rows, nthreads)
        total += dt
        passes += 1
    work = _row_work(case, rows, unit) * passes
    scale = 1e9 if unit == "GB/s" else 1e12
    return work / total / scale, total, used, passes


def cpu_entry(case, oc, rows, unit, what, nthreads=0, min_seconds=3.0):
    v, dt, used, passes = oracle_rate(case, oc, rows, unit, nthreads, min_seconds)
    return {"value": v, "unit": unit, "cores": used, "kind": "oracle",
            "sample": f"{what}: {len(rows)} (token, head) rows x {passes} passes, FP64 oracle, "
                      f"{dt:.1f} s; value = their share of the workload's "
                      f"{'KV bytes' if unit == 'GB/s' else 'useful flops'} / time"}


def oracle_decode_sample(case, min_seconds: float = 10.0, max_passes: int = 4):
    """Times the FP64 oracle on the whole decode batch (every row), repeated
    until about min_seconds of CPU work; returns (GB/s, seconds, threads,
    passes)."""
    s = case.spec
    oc = _oracle_cache(case)
    rows = [[b, h] for b in range(len(s.context_lens)) for h in range(s.num_q_heads)]
    total, passes, used = 0.0, 0, 0
    while passes < max_passes and (passes == 0 or total < min_seconds):
        dt, used = _oracle_rows(oc, case, rows)
        total += dt
        passes += 1
    nbytes = synth.kv_read_bytes(s) * passes
    return nbytes / total / 1e9, total, used, passes


def run_reference(args, rank: int):
    """The reference arm: the FP64 oracle, as it stands, on the host cores.
    Each step is a bounded sample of the decode batch, sized so that W + K
    steps take about REFERENCE_BUDGET_S seconds: `rows_per_step` (sequence,
    query head) rows taken round-robin over the whole batch."""
    if rank != 0:
        return
    spec = synth.workload(DECODE_WORKLOAD)
    case = synth.make_case(spec)
    oc = _oracle_cache(case)
    all_rows = [[b, h] for b in range(len(spec.context_lens)) for h in range(spec.num_q_heads)]
    t_row, used = _oracle_rows(oc, case, all_rows[:8])
    t_row /= 8
    n_calls = max(1, args.warmup + args.steps)
    rows_per_step = int(max(1, min(len(all_rows), REFERENCE_BUDGET_S / n_calls / max(t_row, 1e-6))))
    times = []
    for i in range(n_calls):
        k0 = (i * rows_per_step) % len(all_rows)
        rows = [all_rows[(k0 + r) % len(all_rows)] for r in range(rows_per_step)]
        dt, used = _oracle_rows(oc, case, rows)
        if i >= args.warmup:
            times.append(dt)
    t = sum(times) / len(times)
    val = rows_per_step * _row_bytes(spec) / t / 1e9
    sample = (f"each step: {rows_per_step} of the 256 (sequence, query head) rows of the "
              f"batch-8 x 32K decode, round-robin; FP64 oracle; value = their share of the "
              f"KV bytes / time")
    line = {
        "impl": "reference", "metric": METRIC, "value": val,
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": decode_config(spec, args.gpus),
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- GPU arm --

def new_cache(pk, case, device):
    s = case.spec
    return pk.PagedKVCache.allocate(s.kv_dtype, case.num_blocks, s.block_size, s.num_kv_heads,
                                    s.head_dim, device=device, k_scale=case.k_scale,
                                    v_scale=case.v_scale, scale_per_layer=s.scale_per_layer)


def write_all(pk, cache, case, device, chunk_tokens: int = 1 << 20):
    """Writes every cached token of the case through kv_write_quant (in chunks,
    so that the fp16 sources never all sit on the device)."""
    T = case.k.shape[0]
    for lo in range(0, T, chunk_tokens):
        hi = min(T, lo + chunk_tokens)
        pk.kv_write_quant(cache, case.k[lo:hi].to(device), case.v[lo:hi].to(device),
                          case.slot_mapping[lo:hi].to(device))
    torch.cuda.synchronize()


def build_decode(case, device, copies: int = 2):
    import paged_quantized_kv_quant_b200 as pk
    s = case.spec
    B, ql, Hq, D = len(s.context_lens), s.q_lens[0], s.num_q_heads, s.head_dim
    caches = []
    for _ in range(copies):   # several copies: consecutive calls never share L2 lines
        c = new_cache(pk, case, device)
        write_all(pk, c, case, device)
        caches.append(c)
    new = case.new_token_rows()
    inp = {
        "q": case.q.view(B, ql, Hq, D).to(device),
        "k_new": case.k[new].contiguous().to(device),
        "v_new": case.v[new].contiguous().to(device),
        "slot_new": case.slot_mapping[new].contiguous().to(device),
        "bt": case.block_table.to(device),
        "ctx": case.context_lens.to(device),
    }
    inp["out"] = torch.empty_like(inp["q"])
    max_ctx = max(s.context_lens)
    ws_bytes = pk.decode_workspace_bytes(caches[0], B, ql, Hq, max_ctx)
    inp["ws"] = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    return caches, inp, max_ctx, ws_bytes


def decode_step(pk, cache, inp, max_ctx, scale, write=True, decode=True):
    """write and decode: one appending call; one of them alone: that call."""
    if write and decode:
        q = inp["q"]
        shp = (q.shape[0], q.shape[1], cache.num_kv_heads, q.shape[3])
        pk.paged_attn_decode_append(cache, inp["k_new"].view(shp), inp["v_new"].view(shp), q,
                                    inp["bt"], inp["ctx"], max_ctx, scale, out=inp["out"],
                                    workspace=inp["ws"])
    elif write:
        pk.kv_write_quant(cache, inp["k_new"], inp["v_new"], inp["slot_new"])
    elif decode:
        pk.paged_attn_decode(cache, inp["q"], inp["bt"], inp["ctx"], max_ctx, scale,
                             out=inp["out"], workspace=inp["ws"])


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def time_graphs(graphs, reps, stream, barrier=None, clk=None):
    """Average ms per replay over `reps` replays that cycle through `graphs`,
    bracketed by a barrier and a device synchronize on both sides, CUDA events
    on the launching stream (clock samples taken only meanwhile)."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    if clk:
        clk.resume()
    with torch.cuda.stream(stream):   # replay() launches on the current stream
        e0.record(stream)
        for i in range(reps):
            graphs[i % len(graphs)].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.pause()
    if barrier:
        barrier()
    return e0.elapsed_time(e1) / reps


def time_graphs_min(graphs, stream, clk=None, barrier=None, min_s=MIN_TIMED_S, warm=3):
    """time_graphs over enough replays for at least min_s of device time."""
    with torch.cuda.stream(stream):
        for i in range(warm):
            graphs[i % len(graphs)].replay()
    probe = time_graphs(graphs, max(2, len(graphs)), stream)
    reps = max(len(graphs) * 2, int(math.ceil(min_s * 1e3 / max(probe, 1e-4))))
    reps = (reps + len(graphs) - 1) // len(graphs) * len(graphs)
    return time_graphs(graphs, reps, stream, barrier, clk), reps


def time_graph(graph, reps, stream, barrier=None):
    return time_graphs([graph], reps, stream, barrier)


PROFILES = {
    "decode2": ("decode_b8_ctx32k_fp8_ncu.md",
                ("paged_quantized_kv_quant_b200/csrc/decode.cu",
                 "paged_quantized_kv_quant_b200/csrc/common.cuh",
                 "paged_quantized_kv_quant_b200/csrc/quant.cuh",
                 "paged_quantized_kv_quant_b200/csrc/split_map.cuh")),
    "decode5": ("decode_verify_q5_2x512k_4x256k_int8_ncu.md",
                ("paged_quantized_kv_quant_b200/csrc/decode_tc.cu",
                 "paged_quantized_kv_quant_b200/csrc/kv_stage.cuh",
                 "paged_quantized_kv_quant_b200/csrc/decode.cu",
                 "paged_quantized_kv_quant_b200/csrc/split_map.cuh",
                 "paged_quantized_kv_quant_b200/csrc/common.cuh",
                 "paged_quantized_kv_quant_b200/csrc/tc.cuh")),
    "kvwrite4": ("kv_write_131k_fp8_ncu.md",
                 ("paged_quantized_kv_quant_b200/csrc/kv_write.cu",
                  "paged_quantized_kv_quant_b200/csrc/quant.cuh")),
    "prefill3": ("prefill_8k_causal_fp8_ncu.md",
                 ("paged_quantized_kv_quant_b200/csrc/prefill_tc.cu",
                  "paged_quantized_kv_quant_b200/csrc/common.cuh",
                  "paged_quantized_kv_quant_b200/csrc/kv_stage.cuh",
                  "paged_quantized_kv_quant_b200/csrc/tc.cuh")),
}
DECODE_PROFILE = os.path.join(ROOT, "profiles", PROFILES["decode2"][0])
DECODE_SOURCES = PROFILES["decode2"][1]


def sources_digest(sources) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_sources_digest() -> str:
    return sources_digest(DECODE_SOURCES)


def traffic_from_profile(key: str):
    """DRAM bytes (read + write) of one call of a kernel path from its
    committed ncu summary; None when the summary is missing or was taken on
    other sources than the ones built now."""
    import re
    name, sources = PROFILES[key]
    try:
        with open(os.path.join(ROOT, "profiles", name)) as f:
            text = f.read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_call:\s*([0-9]+)", text)
    d = re.search(r"sources_digest:\s*([0-9a-f]+)", text)
    if not m or not d or d.group(1) != sources_digest(sources):
        return None
    return int(m.group(1))


def decode_traffic_from_profile():
    return traffic_from_profile("decode2")


def reduce_max(x: float, dist=None, device=None) -> float:
    """Max of x over all ranks of the process group (x itself without one):
    every multi-GPU time is the slowest rank's."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, bytes_per_rank: float, ms_max: float) -> float:
    """Whole-job GB/s under weak scaling: every rank reads its own batch's
    bytes in the slowest rank's time."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e9


def run_only(args):
    """W + K calls of one path, nothing else (for profiler captures)."""
    import paged_quantized_kv_quant_b200 as pk
    pk.load_library()
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=device)
    if args.only == "decode":
        spec = synth.workload(args.workload or DECODE_WORKLOAD)
        if args.ctx_div > 1:
            spec.context_lens = [max(spec.block_size, c // args.ctx_div) for c in spec.context_lens]
            spec.name += f"_ctx_div{args.ctx_div}"
        case = synth.make_case(spec)
        # two cache copies alternate when they are small; one copy of a
        # cache larger than L2 already defeats it
        copies = 2 if synth.kv_read_bytes(spec) < (1 << 30) else 1
        caches, inp, max_ctx, _ = build_decode(case, device, copies=copies)
        torch.cuda.empty_cache()   # keep only what the calls use on the device
        calls = [lambda c=c: decode_step(pk, c, inp, max_ctx, case.softmax_scale, write=False)
                 for c in caches]
    elif args.only == "kv_write":
        # the KV write of every cached token of a prefill workload, as the
        # prefill secondaries time it
        spec = synth.workload(args.workload or PREFILL_WORKLOAD)
        case = synth.make_case(spec)
        c = new_cache(pk, case, device)
        kd, vd = case.k.to(device), case.v.to(device)
        smd = case.slot_mapping.to(device)
        calls = [lambda: pk.kv_write_quant(c, kd, vd, smd)]
    else:
        spec = synth.workload(args.workload or PREFILL_WORKLOAD)
        case = synth.make_case(spec)
        c = new_cache(pk, case, device)
        write_all(pk, c, case, device)
        q = case.q.to(device)
        out = torch.empty_like(q)
        cu, bt, ctx = (case.cu_seqlens_q.to(device), case.block_table.to(device),
                       case.context_lens.to(device))
        mq = max(spec.q_lens)
        calls = [lambda: pk.paged_attn_prefill(c, q, cu, bt, ctx, mq, case.softmax_scale,
                                               out=out)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(max(0, args.warmup)):
            calls[i % len(calls)]()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(max(1, args.steps)):
            calls[i % len(calls)]()
        e1.record(stream)
    torch.cuda.synchronize()
    print(json.dumps({"only": args.only, "workload": spec.name, "calls": max(1, args.steps),
                      "ms_per_call": e0.elapsed_time(e1) / max(1, args.steps)}), flush=True)


# ------------------------------------------------------------ secondaries --

def sec_decode(pk, n, device, stream, clk, hbm_peak, peak_src, copies=None):
    """Decode workload n (1 or 5): KV GB/s of one call against HBM.  Enough
    cache copies alternate that the inputs exceed L2."""
    spec = synth.workload(n)
    case = synth.make_case(spec)
    kvb = synth.kv_read_bytes(spec)
    if copies is None:
        copies = max(1, int(math.ceil(160e6 / kvb)))   # > 126 MB of L2 in total
    caches, inp, max_ctx, _ = build_decode(case, device, copies=copies)
    sc = case.softmax_scale
    with torch.cuda.stream(stream):
        for c in caches:
            decode_step(pk, c, inp, max_ctx, sc, write=False)
    torch.cuda.synchronize()
    graphs = [capture(lambda c=c: decode_step(pk, c, inp, max_ctx, sc, write=False), stream)
              for c in caches]
    ms, reps = time_graphs_min(graphs, stream, clk)
    gbs = kvb / (ms * 1e-3) / 1e9
    entry = {"workload": spec.name, "metric": "decode KV-read GB/s", "value": gbs,
             "unit": "GB/s", "us_per_call": ms * 1e3, "timed_calls": reps,
             "algorithmic_bytes": kvb,
             "l2": f"{copies} cache copies alternated ({copies * kvb / 1e6:.0f} MB)",
             "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                          "frac": gbs / hbm_peak, "peak_source": peak_src,
                          "traffic": traffic_from_profile("decode5") if n == 5 else None}}
    del graphs, caches, inp
    torch.cuda.empty_cache()
    return entry, case


def sec_prefill(pk, n, device, stream, clk, bf16_peak, hbm_peak, peak_src):
    """Prefill workload n (3 or 4): useful TFLOP/s of one call against the
    measured dense 16-bit tensor peak, and the KV write of all its tokens."""
    spec = synth.workload(n)
    case = synth.make_case(spec)
    c = new_cache(pk, case, device)
    T = case.k.shape[0]
    kd, vd, smd = case.k.to(device), case.v.to(device), case.slot_mapping.to(device)
    q = case.q.to(device)
    out = torch.empty_like(q)
    cu, bt, ctx = (case.cu_seqlens_q.to(device), case.block_table.to(device),
                   case.context_lens.to(device))
    mq = max(spec.q_lens)
    sc = case.softmax_scale
    with torch.cuda.stream(stream):
        pk.kv_write_quant(c, kd, vd, smd)
        pk.paged_attn_prefill(c, q, cu, bt, ctx, mq, sc, out=out)
    torch.cuda.synchronize()
    g_pf = capture(lambda: pk.paged_attn_prefill(c, q, cu, bt, ctx, mq, sc, out=out), stream)
    g_wr = capture(lambda: pk.kv_write_quant(c, kd, vd, smd), stream)
    ms_pf, reps_pf = time_graphs_min([g_pf], stream, clk)
    ms_wr, reps_wr = time_graphs_min([g_wr], stream, clk)
    flops = synth.useful_flops(spec)
    tf = flops / (ms_pf * 1e-3) / 1e12
    wbytes = T * spec.num_kv_heads * spec.head_dim * (2 * 2 + 2)   # fp16 K,V in; codes out
    wgbs = wbytes / (ms_wr * 1e-3) / 1e9
    entry = {"workload": spec.name, "metric": "causal prefill useful TFLOP/s", "value": tf,
             "unit": "TFLOP/s", "ms": ms_pf, "timed_calls": reps_pf, "useful_flop": flops,
             "frac_of_bf16_peak": tf / bf16_peak, "peak": bf16_peak, "peak_source": peak_src,
             "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16_peak,
                          "unit": "TFLOP/s", "frac": tf / bf16_peak, "peak_source": peak_src,
                          "traffic": traffic_from_profile("prefill3") if n == 3 else None}}
    wentry = {"workload": f"kv_write_quant of {spec.name} ({T} tokens)", "value": wgbs,
              "unit": "GB/s", "ms": ms_wr, "timed_calls": reps_wr, "bytes": wbytes,
              "frac": wgbs / hbm_peak,
              "roofline": {"bound": "hbm", "achieved": wgbs, "peak": hbm_peak, "unit": "GB/s",
                           "frac": wgbs / hbm_peak, "peak_source": peak_src,
                           "traffic": traffic_from_profile("kvwrite4") if n == 4 else None}}
    del g_pf, g_wr, c, kd, vd, smd, q, out
    torch.cuda.empty_cache()
    return entry, wentry, case


def sec_format_decode(pk, kv_dtype, device, stream, clk, hbm_peak, peak_src):
    """The batch-8 x 32K decode with another cache format (E5M2: the same
    bytes as E4M3; FP16: twice as many): KV GB/s of one call."""
    base = synth.workload(DECODE_WORKLOAD)
    name = {synth.FP8_E5M2: "e5m2", synth.FP16: "fp16"}[kv_dtype]
    spec = synth.CaseSpec("decode", kv_dtype, base.num_q_heads, base.num_kv_heads,
                          base.context_lens, base.q_lens, outlier_frac=base.outlier_frac,
                          seed=base.seed, name=base.name.replace("e4m3", name))
    case = synth.make_case(spec)
    kvb = synth.kv_read_bytes(spec)
    caches, inp, max_ctx, _ = build_decode(case, device, copies=2)
    sc = case.softmax_scale
    with torch.cuda.stream(stream):
        for c in caches:
            decode_step(pk, c, inp, max_ctx, sc, write=False)
    torch.cuda.synchronize()
    graphs = [capture(lambda c=c: decode_step(pk, c, inp, max_ctx, sc, write=False), stream)
              for c in caches]
    ms, reps = time_graphs_min(graphs, stream, clk)
    gbs = kvb / (ms * 1e-3) / 1e9
    del graphs, caches, inp
    torch.cuda.empty_cache()
    return {"workload": spec.name, "metric": "decode KV-read GB/s", "value": gbs, "unit": "GB/s",
            "us_per_call": ms * 1e3, "timed_calls": reps, "algorithmic_bytes": kvb,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "peak_source": peak_src, "traffic": None}}


def sec_block_copy(pk, device, stream, clk):
    """KV page copies between the GPU pool and a pinned host tier (E4M3 cache of
    the batch-8 x 32K shape, 1 GiB of blocks each way), against a plain pinned
    copy of the same bytes measured in the same run."""
    nb, bs, hkv = 65536, 16, 4
    blk_bytes = 2 * hkv * bs * 128                    # K and V of one block
    dev = pk.PagedKVCache.allocate(synth.FP8_E4M3, nb, bs, hkv, device=device,
                                   k_scale=[1.0] * hkv, v_scale=[1.0] * hkv)
    host = pk.PagedKVCache.allocate(synth.FP8_E4M3, nb, bs, hkv, device="cpu", pin_host=True,
                                    k_scale=[1.0] * hkv, v_scale=[1.0] * hkv)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(0)).to(torch.int32)
    out_pairs = torch.stack([torch.arange(nb, dtype=torch.int32), perm], 1).to(device)
    in_pairs = torch.stack([perm, torch.arange(nb, dtype=torch.int32)], 1).to(device)
    with torch.cuda.stream(stream):
        pk.kv_copy_blocks(host, dev, out_pairs)
        pk.kv_copy_blocks(dev, host, in_pairs)
    torch.cuda.synchronize()
    g_out = capture(lambda: pk.kv_copy_blocks(host, dev, out_pairs), stream)
    g_in = capture(lambda: pk.kv_copy_blocks(dev, host, in_pairs), stream)
    ms_out, _ = time_graphs_min([g_out], stream, clk, min_s=0.5)
    ms_in, _ = time_graphs_min([g_in], stream, clk, min_s=0.5)
    # reference: one contiguous pinned copy of the same bytes each way
    flat_d, flat_h = dev.k_cache.view(-1), host.k_cache.view(-1)
    with torch.cuda.stream(stream):
        flat_h.copy_(flat_d, non_blocking=True)
    torch.cuda.synchronize()
    g_d2h = capture(lambda: (host.k_cache.copy_(dev.k_cache, non_blocking=True),
                             host.v_cache.copy_(dev.v_cache, non_blocking=True)), stream)
    g_h2d = capture(lambda: (dev.k_cache.copy_(host.k_cache, non_blocking=True),
                             dev.v_cache.copy_(host.v_cache, non_blocking=True)), stream)
    ms_d2h, _ = time_graphs_min([g_d2h], stream, clk, min_s=0.5)
    ms_h2d, _ = time_graphs_min([g_h2d], stream, clk, min_s=0.5)
    total = nb * blk_bytes
    gbs = lambda ms: total / (ms * 1e-3) / 1e9
    del g_out, g_in, g_d2h, g_h2d, dev, host
    torch.cuda.empty_cache()
    return {"workload": f"kv_copy_blocks, {nb} E4M3 blocks of 16 tokens x 4 heads "
                        f"({total >> 20} MiB) in a random order, GPU pool <-> pinned host tier",
            "metric": "page copy GB/s", "unit": "GB/s",
            "to_host": {"value": gbs(ms_out), "ms": ms_out,
                        "frac_of_pinned_memcpy": ms_d2h / ms_out},
            "to_device": {"value": gbs(ms_in), "ms": ms_in,
                          "frac_of_pinned_memcpy": ms_h2d / ms_in},
            "pinned_memcpy_gbs": {"d2h": gbs(ms_d2h), "h2d": gbs(ms_h2d)},
            "roofline": {"bound": "host link", "peak": "a contiguous pinned cudaMemcpy of the "
                                                       "same bytes, measured in this run"}}


def prefill_sample_rows(case, n_rows, seed):
    """Random (token, head) rows of a prefill chunk, spread over the whole chunk."""
    rng = np.random.default_rng(seed)
    s = case.spec
    total = int(case.cu_seqlens_q[-1])
    return np.stack([rng.integers(total, size=n_rows), rng.integers(s.num_q_heads, size=n_rows)],
                    1).astype(np.int32)


def main():
    args = parse()
    if args.only:
        run_only(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", local if world > 1 else 0)
    import paged_quantized_kv_quant_b200 as pk
    pk.load_library()
    hbm_peak, bf16_peak, bf16_sus, peak_src = peaks()

    barrier = (lambda: dist.barrier()) if dist else None

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dist, device)

    clk = ClockSampler(device.index)
    clk.pause()
    clk.__enter__()

    # ---------------- decode workload ----------------
    spec = synth.workload(DECODE_WORKLOAD)
    case = synth.make_case(spec)
    caches, inp, max_ctx, ws_bytes = build_decode(case, device)
    scale = case.softmax_scale
    kv_bytes = synth.kv_read_bytes(spec)
    plan_splits = ws_bytes > 0
    stream = torch.cuda.Stream(device=device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for c in caches:        # warm up library state (function attributes, maps) outside capture
            decode_step(pk, c, inp, max_ctx, scale)
    torch.cuda.synchronize()
    # one graph per cache copy: consecutive steps alternate the copies
    g_step = [capture(lambda c=c: decode_step(pk, c, inp, max_ctx, scale), stream)
              for c in caches]
    g_dec = [capture(lambda c=c: decode_step(pk, c, inp, max_ctx, scale, write=False), stream)
             for c in caches]
    g_wr = [capture(lambda c=c: decode_step(pk, c, inp, max_ctx, scale, decode=False), stream)
            for c in caches]
    steps = max(1, args.steps)
    with torch.cuda.stream(stream):
        for i in range(max(0, args.warmup)):
            g_step[i % 2].replay()
    torch.cuda.synchronize()
    ms_step = max_over_ranks(time_graphs(g_step, steps, stream, barrier, clk))
    # per-kernel timing (same graphs, same inputs), each over >= MIN_TIMED_S
    ms_dec, reps_dec = time_graphs_min(g_dec, stream, clk, barrier)
    ms_dec = max_over_ranks(ms_dec)
    ms_wr, _ = time_graphs_min(g_wr, stream, clk, barrier)
    ms_wr = max_over_ranks(ms_wr)
    value = job_throughput(world, kv_bytes, ms_step)
    dec_gbs = kv_bytes / (ms_dec * 1e-3) / 1e9

    # ---------------- end to end through the public API, host buffers ----------------
    # Every step uploads its inputs (new token's K/V, Q, block table, context
    # lengths) from pinned host memory and reads its output back.  The
    # inputs sit back to back in one pinned buffer, so one copy moves them; two
    # device copies of that buffer (and of the output) let step i+1's upload
    # and step i's download run on their own streams while step i computes.
    names = ("q", "k_new", "v_new", "bt", "ctx")
    offs, total = {}, 0
    for k in names:
        nb = inp[k].numel() * inp[k].element_size()
        offs[k] = (total, nb)
        total += (nb + 255) // 256 * 256
    host_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for k, (o, nb) in offs.items():
        host_in[o:o + nb].copy_(inp[k].reshape(-1).view(torch.uint8).cpu())
    dev_in = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
    views = [{k: buf[o:o + nb].view(inp[k].dtype).view(inp[k].shape)
              for k, (o, nb) in offs.items()} for buf in dev_in]
    dev_out = [torch.empty_like(inp["out"]) for _ in range(2)]
    host_out = [torch.empty(inp["out"].shape, dtype=inp["out"].dtype).pin_memory()
                for _ in range(2)]
    h2d = sum(nb for _, nb in offs.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        if i >= 2:
            up.wait_event(done[b])           # step i-2 finished with this input buffer
        with torch.cuda.stream(up):
            dev_in[b].copy_(host_in, non_blocking=True)
        copied[b].record(up)
        stream.wait_event(copied[b])
        if i >= 2:
            stream.wait_event(read[b])       # step i-2's output has been read back
        d = views[b]
        shp = (d["q"].shape[0], d["q"].shape[1], caches[0].num_kv_heads, d["q"].shape[3])
        pk.paged_attn_decode_append(caches[i % 2], d["k_new"].view(shp), d["v_new"].view(shp),
                                    d["q"], d["bt"], d["ctx"], max_ctx, scale, out=dev_out[b],
                                    workspace=inp["ws"], stream=stream)
        done[b].record(stream)
        down.wait_event(done[b])
        with torch.cuda.stream(down):
            host_out[b].copy_(dev_out[b], non_blocking=True)
        read[b].record(down)

    def e2e_steps(n):
        up.wait_stream(stream)
        down.wait_stream(stream)
        for i in range(n):
            e2e_step(i)
        stream.wait_stream(up)
        stream.wait_stream(down)

    # The loop is captured once in a CUDA graph of E2E_GRAPH_STEPS steps (the
    # uploads and downloads become memcpy nodes on the forked streams), as a
    # serving loop would, so the host's per-call overhead is not what is timed.
    with torch.cuda.stream(stream):
        e2e_steps(4)
    torch.cuda.synchronize()
    g_e2e = capture(lambda: e2e_steps(E2E_GRAPH_STEPS), stream)
    n_rep = max(1, args.e2e_steps // E2E_GRAPH_STEPS)
    n_e2e = n_rep * E2E_GRAPH_STEPS
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_e2e.replay()
    ms_e2e = max_over_ranks(time_graph(g_e2e, n_rep, stream, barrier) / E2E_GRAPH_STEPS)
    e2e_val = job_throughput(world, kv_bytes, ms_e2e)
    ok_out = bool(torch.equal(host_out[(n_e2e - 1) % 2].to(device), dev_out[(n_e2e - 1) % 2]))
    del g_step, g_dec, g_wr, g_e2e, dev_in, dev_out
    caches_keep = caches
    del caches
    torch.cuda.empty_cache()

    # ---------------- the other four workloads ----------------
    secondary = None
    cases = {DECODE_WORKLOAD: case}
    if not args.no_prefill:
        del caches_keep
        torch.cuda.empty_cache()
        secondary = {}
        e1, cases[1] = sec_decode(pk, 1, device, stream, clk, hbm_peak, peak_src)
        e3, w3, cases[3] = sec_prefill(pk, 3, device, stream, clk, bf16_peak, hbm_peak, peak_src)
        e4, w4, cases[4] = sec_prefill(pk, 4, device, stream, clk, bf16_peak, hbm_peak, peak_src)
        e5, cases[5] = sec_decode(pk, 5, device, stream, clk, hbm_peak, peak_src)
        secondary = {"decode_1x1k": e1, "prefill": e3, "chunked_prefill": e4,
                     "verify_decode": e5, "kv_write_8k": w3, "kv_write_131k": w4,
                     "decode_e5m2": sec_format_decode(pk, synth.FP8_E5M2, device, stream, clk,
                                                      hbm_peak, peak_src),
                     "decode_fp16": sec_format_decode(pk, synth.FP16, device, stream, clk,
                                                      hbm_peak, peak_src),
                     "block_copy": sec_block_copy(pk, device, stream, clk)}
    clk.__exit__()

    # ---------------- CPU baseline (oracle, rank 0, N = 1) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, dt, used, passes = oracle_decode_sample(case)
        cpu = {"value": gbs, "unit": "GB/s", "cores": used, "kind": "oracle",
               "sample": f"the whole batch-8 x 32K decode (all 256 rows, 268,435,456 KV "
                         f"bytes) x {passes} passes, FP64 oracle, {dt:.1f} s"}
        oc2 = _oracle_cache(case)
        cpu_1core = cpu_entry(case, oc2, [[b, 0] for b in range(8)], "GB/s",
                              "batch-8 x 32K decode, head 0 of every sequence", nthreads=1)
        cpu["single_core"] = cpu_1core
        del oc2
        if secondary:
            c1 = cases[1]
            oc = _oracle_cache(c1)
            rows1 = [[0, h] for h in range(c1.spec.num_q_heads)]
            secondary["decode_1x1k"]["cpu_baseline"] = cpu_entry(
                c1, oc, rows1, "GB/s", "the whole 1 x 1K decode")
            secondary["decode_1x1k"]["cpu_baseline"]["single_core"] = cpu_entry(
                c1, oc, rows1, "GB/s", "the whole 1 x 1K decode", nthreads=1)
            c3 = cases[3]
            oc = _oracle_cache(c3)
            rows3 = prefill_sample_rows(c3, 256, 3)
            secondary["prefill"]["cpu_baseline"] = cpu_entry(
                c3, oc, rows3, "TFLOP/s", "8K causal prefill, random rows")
            secondary["prefill"]["cpu_baseline"]["single_core"] = cpu_entry(
                c3, oc, rows3[:16], "TFLOP/s", "8K causal prefill, random rows", nthreads=1)
            c4 = cases[4]
            oc = _oracle_cache(c4)
            secondary["chunked_prefill"]["cpu_baseline"] = cpu_entry(
                c4, oc, prefill_sample_rows(c4, 64, 4), "TFLOP/s",
                "8K chunk over a 120K prefix, random rows")
            c5 = cases[5]
            oc = _oracle_cache(c5, only_seqs=[2])      # one 256K sequence of the six
            rows5 = [[2 * 5 + t, h] for t in range(5) for h in range(0, 32, 4)]
            secondary["verify_decode"]["cpu_baseline"] = cpu_entry(
                c5, oc, rows5, "GB/s", "verify decode, one 256K sequence, 5 tokens x 8 heads")
            del oc

    launches_per_step = 1 + (1 if plan_splits else 0)   # appending split kernel (+ merge)
    traffic = decode_traffic_from_profile()
    line = {
        "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 (E4M3 codes dequantised to f16, f32 accumulate)",
        "data": "synthetic (seeded N(0,1), 1% channels x8)",
        "config": decode_config(spec, world),
        "clocks": clk.summary(),
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                "pipelining": "per step one pinned upload (own stream) and one download (third "
                              "stream), double-buffered device inputs/outputs; 8 steps per "
                              "CUDA graph replay",
                "last_output_read_back_matches": ok_out},
        "gpu_launches": launches_per_step * steps,
        "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": dec_gbs / hbm_peak, "traffic": traffic,
                     "kernel": "pkvq_paged_attn_decode (split + merge kernels)",
                     "ms_per_launch": ms_dec, "timed_calls": reps_dec,
                     "algorithmic_bytes": kv_bytes, "peak_source": peak_src},
        "kv_write_ms": ms_wr,
        "cpu_baseline": cpu,
        "secondary": secondary,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
