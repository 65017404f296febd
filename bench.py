#!/usr/bin/env python
"""Benchmark: paged 8-bit-KV attention on B200.

One step = one decode step of the batch-8 workload (8 sequences x 32,768
cached tokens, 32 query / 4 KV heads, head_dim 128, block 16, FP8 E4M3 cache
with per-KV-head scales, 1% outlier channels x8): write + quantize the step's
new token into the paged cache (pkvq_kv_write_quant), then attend over the
whole cache (pkvq_paged_attn_decode: split kernel + merge kernel).  The metric
is KV-read GB/s: the K and V code bytes one step must read (268,435,456 B per
GPU) divided by the step time.  Causal prefill TFLOP/s (8,192-token prefill,
same heads) is reported beside it under "secondary".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pkvq|reference]
    python bench.py --only decode|prefill [--steps K] [--warmup W]

--only runs nothing but W + K calls of one kernel path on its workload (the
decode call on the batch-8 x 32K cache, or the 8K causal prefill) and prints
their average time: the command the ncu captures are taken with.

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
            "step": "kv_write_quant(new token) + paged_attn_decode",
            "l2": "inputs larger than L2: two 268 MB caches alternated step by step",
            "parallelism": f"dp{world} (independent batches per GPU)"}
PREFILL_WORKLOAD = 3
REFERENCE_BUDGET_S = 120.0
E2E_GRAPH_STEPS = 8
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["pkvq", "reference"], default="pkvq")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--only", choices=["decode", "prefill"], default=None)
    ap.add_argument("--workload", type=int, default=None,
                    help="with --only: the named workload to run (decode 1, 2, 5; prefill 3, 4)")
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
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ CPU oracle --

def _bits16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_cache(case):
    import oracle
    s = case.spec
    oc = oracle.Cache(s.kv_dtype, case.num_blocks, s.block_size, s.num_kv_heads, s.head_dim,
                      None if case.k_scale is None else case.k_scale.numpy(),
                      None if case.v_scale is None else case.v_scale.numpy())
    oc.write(_bits16(case.k), _bits16(case.v), case.slot_mapping.numpy())
    return oc


def _oracle_rows(oc, case, rows):
    """One oracle pass over the given (sequence, query head) rows; seconds, threads."""
    import oracle
    t0 = time.perf_counter()
    _, _, used = oracle.paged_attention(oc, _bits16(case.q), case.cu_seqlens_q.numpy(),
                                        case.context_lens.numpy(), case.block_table.numpy(),
                                        case.softmax_scale,
                                        rows=np.asarray(rows, np.int32).reshape(-1, 2))
    return time.perf_counter() - t0, used


def _row_bytes(spec) -> float:
    """Algorithmic KV bytes per (sequence, query head) row: a 1/Hq share of
    its sequence's KV bytes (the G rows of a KV head read the same codes)."""
    return synth.kv_read_bytes(spec) / len(spec.context_lens) / spec.num_q_heads


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

def build_decode(case, device, copies: int = 2):
    import paged_quantized_kv_quant_b200 as pk
    s = case.spec
    B, ql, Hq, D = len(s.context_lens), s.q_lens[0], s.num_q_heads, s.head_dim
    k_all, v_all = case.k.to(device), case.v.to(device)
    sm_all = case.slot_mapping.to(device)
    caches = []
    for _ in range(copies):   # two copies: consecutive steps never share L2 lines
        c = pk.PagedKVCache.allocate(s.kv_dtype, case.num_blocks, s.block_size,
                                     s.num_kv_heads, D, device=device,
                                     k_scale=case.k_scale, v_scale=case.v_scale)
        pk.kv_write_quant(c, k_all, v_all, sm_all)
        caches.append(c)
    del k_all, v_all, sm_all
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
    inp["ws"] = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    return caches, inp, max_ctx, ws_bytes


def decode_step(pk, cache, inp, max_ctx, scale, write=True, decode=True):
    if write:
        pk.kv_write_quant(cache, inp["k_new"], inp["v_new"], inp["slot_new"])
    if decode:
        pk.paged_attn_decode(cache, inp["q"], inp["bt"], inp["ctx"], max_ctx, scale,
                             out=inp["out"], workspace=inp["ws"])


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def time_graph(graph, reps, stream, barrier=None):
    """Average ms per replay over `reps` replays, bracketed by a barrier and a
    device synchronize on both sides, CUDA events on the launching stream."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):   # replay() launches on the current stream
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return e0.elapsed_time(e1) / reps


DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_b8_ctx32k_fp8_ncu.md")
DECODE_SOURCES = ("paged_quantized_kv_quant_b200/csrc/decode.cu",
                  "paged_quantized_kv_quant_b200/csrc/common.cuh")


def decode_sources_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


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


def decode_traffic_from_profile():
    """DRAM bytes (read + write) of one decode call, split and merge kernels,
    from the committed ncu summary; None when the summary is missing or was
    taken on other decode sources than the ones built now."""
    import re
    try:
        with open(DECODE_PROFILE) as f:
            text = f.read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_call:\s*([0-9]+)", text)
    d = re.search(r"decode_sources_digest:\s*([0-9a-f]+)", text)
    if not m or not d or d.group(1) != decode_sources_digest():
        return None
    return int(m.group(1))


def run_only(args):
    """W + K calls of one path, nothing else (for profiler captures)."""
    import paged_quantized_kv_quant_b200 as pk
    pk.load_library()
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=device)
    if args.only == "decode":
        spec = synth.workload(args.workload or DECODE_WORKLOAD)
        case = synth.make_case(spec)
        # two cache copies alternate when they are small; one copy of a
        # cache larger than L2 already defeats it
        copies = 2 if synth.kv_read_bytes(spec) < (1 << 30) else 1
        caches, inp, max_ctx, _ = build_decode(case, device, copies=copies)
        torch.cuda.empty_cache()   # keep only what the calls use on the device
        calls = [lambda c=c: decode_step(pk, c, inp, max_ctx, case.softmax_scale, write=False)
                 for c in caches]
    else:
        spec = synth.workload(args.workload or PREFILL_WORKLOAD)
        case = synth.make_case(spec)
        c = pk.PagedKVCache.allocate(spec.kv_dtype, case.num_blocks, spec.block_size,
                                     spec.num_kv_heads, device=device,
                                     k_scale=case.k_scale, v_scale=case.v_scale)
        pk.kv_write_quant(c, case.k.to(device), case.v.to(device), case.slot_mapping.to(device))
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
    g_step = capture(lambda: [decode_step(pk, c, inp, max_ctx, scale) for c in caches], stream)
    g_dec = capture(lambda: [decode_step(pk, c, inp, max_ctx, scale, write=False) for c in caches],
                    stream)
    g_wr = capture(lambda: [decode_step(pk, c, inp, max_ctx, scale, decode=False) for c in caches],
                   stream)
    reps = max(1, args.steps // 2)
    steps = 2 * reps
    warm = max(2, (args.warmup + 1) // 2)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g_step.replay()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        ms_pair = time_graph(g_step, reps, stream, barrier)
    ms_step = max_over_ranks(ms_pair / 2)
    # per-kernel timing (same graphs, same inputs): decode call alone, write alone
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g_dec.replay()
    ms_dec = max_over_ranks(time_graph(g_dec, reps, stream, barrier) / 2)
    ms_wr = max_over_ranks(time_graph(g_wr, reps, stream, barrier) / 2)
    value = job_throughput(world, kv_bytes, ms_step)
    dec_gbs = kv_bytes / (ms_dec * 1e-3) / 1e9

    # ---------------- end to end through the public API, host buffers ----------------
    # Every step uploads its inputs (new token's K/V and slots, Q, block table,
    # context lengths) from pinned host memory and reads its output back.  The
    # inputs sit back to back in one pinned buffer, so one copy moves them; two
    # device copies of that buffer (and of the output) let step i+1's upload
    # and step i's download run on their own streams while step i computes.
    names = ("q", "k_new", "v_new", "slot_new", "bt", "ctx")
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
        pk.kv_write_quant(caches[i % 2], d["k_new"], d["v_new"], d["slot_new"], stream=stream)
        pk.paged_attn_decode(caches[i % 2], d["q"], d["bt"], d["ctx"], max_ctx, scale,
                             out=dev_out[b], workspace=inp["ws"], stream=stream)
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

    # ---------------- secondary: causal prefill 8K ----------------
    secondary = None
    if not args.no_prefill:
        pspec = synth.workload(PREFILL_WORKLOAD)
        pcase = synth.make_case(pspec)
        pc = pk.PagedKVCache.allocate(pspec.kv_dtype, pcase.num_blocks, pspec.block_size,
                                      pspec.num_kv_heads, device=device,
                                      k_scale=pcase.k_scale, v_scale=pcase.v_scale)
        pk_, pv_ = pcase.k.to(device), pcase.v.to(device)
        psm = pcase.slot_mapping.to(device)
        pq = pcase.q.to(device)
        pout = torch.empty_like(pq)
        pcu, pbt, pctx = (pcase.cu_seqlens_q.to(device), pcase.block_table.to(device),
                          pcase.context_lens.to(device))
        mq = max(pspec.q_lens)
        with torch.cuda.stream(stream):
            pk.kv_write_quant(pc, pk_, pv_, psm)
            pk.paged_attn_prefill(pc, pq, pcu, pbt, pctx, mq, pcase.softmax_scale, out=pout)
        torch.cuda.synchronize()
        g_pf = capture(lambda: pk.paged_attn_prefill(pc, pq, pcu, pbt, pctx, mq,
                                                     pcase.softmax_scale, out=pout), stream)
        g_pw = capture(lambda: pk.kv_write_quant(pc, pk_, pv_, psm), stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g_pf.replay()
        preps = 20
        ms_pf = max_over_ranks(time_graph(g_pf, preps, stream, barrier))
        ms_pw = max_over_ranks(time_graph(g_pw, preps, stream, barrier))
        flops = synth.useful_flops(pspec)
        wbytes = pcase.k.numel() * 2 * 2 + pcase.k.numel() * 2   # fp16 in, codes out
        secondary = {
            "prefill": {"workload": pspec.name, "metric": "causal prefill useful TFLOP/s",
                        "value": flops / (ms_pf * 1e-3) / 1e12, "unit": "TFLOP/s",
                        "ms": ms_pf, "useful_flop": flops,
                        "frac_of_bf16_peak": flops / (ms_pf * 1e-3) / 1e12 / bf16_peak,
                        "peak": bf16_peak, "peak_source": peak_src},
            "kv_write_8k": {"value": wbytes / (ms_pw * 1e-3) / 1e9, "unit": "GB/s",
                            "ms": ms_pw, "bytes": wbytes,
                            "frac": wbytes / (ms_pw * 1e-3) / 1e9 / hbm_peak},
        }
        del pc, pk_, pv_

    # ---------------- CPU baseline (oracle, rank 0, N = 1) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, dt, used, passes = oracle_decode_sample(case)
        cpu = {"value": gbs, "unit": "GB/s", "cores": used, "kind": "oracle",
               "sample": f"the whole batch-8 x 32K decode (all 256 rows, 268,435,456 KV "
                         f"bytes) x {passes} passes, FP64 oracle, {dt:.1f} s"}

    launches_per_step = 2 + (1 if plan_splits else 0)
    traffic = decode_traffic_from_profile()
    line = {
        "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": 2 * warm,
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
                     "ms_per_launch": ms_dec, "algorithmic_bytes": kv_bytes,
                     "peak_source": peak_src},
        "kv_write_ms": ms_wr,
        "cpu_baseline": cpu,
        "secondary": secondary,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_step, g_dec, g_wr, g_e2e
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
