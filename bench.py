#!/usr/bin/env python
"""Throughput of the DSA forward pass (indexer -> top-k -> sparse MLA attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one whole forward pass over one batch of synthetic input of the chosen
workload, with inputs resident in HBM.  Prints ONE JSON line (rank 0).

  value      tokens/s over all ranks (query rows processed / max-over-ranks device time)
  e2e        same metric through the public API with pinned host buffers; the H2D copy
             of the step's inputs and the D2H copy of its outputs are inside the timing
  roofline   the dominant kernel: algorithmic FLOPs (or bytes) per launch / its mean
             CUDA-event duration, against the measured peak in MEASURED_PEAKS.json
  stages     the same for every kernel of the step
  workloads  the other workloads the metric names (decode at 128K context; 128K prefill
             in 4096-query chunks), measured the same way with fewer steps; and the
             indexer's training loss (forward) on the headline step's own outputs
  cpu_baseline  the fp64 oracle on a bounded sample of the headline workload, host cores

Multi-GPU (torchrun): every rank runs its own independent problem (weak scaling, no
collective on the data path); a barrier and CUDA synchronisation bracket the timed
region and the slowest rank's time is used.
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
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dsa_inputs import WORKLOADS, make_inputs, make_key_side, make_query_side  # noqa: E402

METRIC = "DSA tokens/s (prefill 32K/128K, decode@128K ctx); % of FP8 peak / HBM roofline"
HEADLINE = "prefill_32k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------ setup

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--no-extra", action="store_true", help="skip the supplementary workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--loss", action="store_true", help="time the indexer loss even with --no-extra")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-fp8-peak", action="store_true", help="skip measuring the FP8 GEMM peak")
    ap.add_argument("--stage", choices=["forward", "indexer_topk"], default="forward",
                    help="indexer_topk: time only the fused indexer + top-k of the workload (profiling runs); "
                         "prints its own JSON line")
    return ap.parse_args()


def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "ours" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, local, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dsa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def measure_fp8_peak(device="cuda", n=8192, sustain_s=2.0):
    """Dense FP8 (e4m3 x e4m3, fp32 accumulate) GEMM throughput of this GPU through
    cuBLASLt (torch._scaled_mm), M = N = K = n, in TFLOP/s.

    burst: the best of 10 single calls after warm-up (for a kernel timed alone);
    sustained: back-to-back calls for about ``sustain_s`` seconds (for a kernel
    timed inside a long step, under the power cap).  Both accumulation modes of
    the library are tried and the faster is kept.  No clock or power setting is
    touched."""
    g = torch.Generator(device=device).manual_seed(1234)
    a = torch.randn(n, n, device=device, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=device, generator=g).to(torch.float8_e4m3fn).t()   # column-major operand
    one = torch.ones((), device=device, dtype=torch.float32)
    flops = 2.0 * n ** 3
    best_ms, mode = float("inf"), None
    for fast in (False, True):
        def mm():
            return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16, use_fast_accum=fast)
        for _ in range(3):
            mm()
        torch.cuda.synchronize()
        for _ in range(10):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            mm()
            e.record()
            e.synchronize()
            ms = s.elapsed_time(e)
            if ms < best_ms:
                best_ms, mode = ms, fast
    def mm():
        return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16, use_fast_accum=mode)
    iters = max(10, int(sustain_s / (best_ms * 1e-3)))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(iters):
        mm()
    e.record()
    e.synchronize()
    sus_ms = s.elapsed_time(e) / iters
    del a, b
    torch.cuda.empty_cache()
    return {"fp8_tflops": flops / (best_ms * 1e-3) / 1e12, "fp8_tflops_sustained": flops / (sus_ms * 1e-3) / 1e12,
            "method": f"torch._scaled_mm e4m3 {n}^3 (cuBLASLt), use_fast_accum={mode}; burst = best of 10, "
                      f"sustained = mean of {iters} back-to-back calls"}


# ------------------------------------------------------------------------------------ work model

def work_model(wl, Lq=None, q_offset=None):
    """Algorithmic work of one forward over queries [q_offset, q_offset+Lq) (per batch), x B."""
    Lq = wl.Lq if Lq is None else Lq
    q0 = wl.q_offset if q_offset is None else q_offset
    first, last = q0 + 1, q0 + Lq
    causal = (first + last) * Lq // 2 * wl.B
    t = np.arange(q0, q0 + Lq, dtype=np.int64)
    selected = int(np.minimum(wl.k, t + 1).sum()) * wl.B
    rows = wl.B * Lq
    return {
        "rows": rows,
        "causal_pairs": causal,
        "selected_pairs": selected,
        # indexer: one FP8 dot of width d_I per (pair, head); bytes: keys + scales and
        # the query side read once, the causal scores written (staged selection)
        "indexer_flops": 2.0 * causal * wl.H_I * wl.d_I,
        "indexer_bytes": wl.B * (q0 + Lq) * (wl.d_I + 4) + rows * wl.H_I * (wl.d_I + 2) + causal * 4.0,
        # top-k: the causal scores read once, the selected indices written
        "topk_bytes": causal * 4.0 + rows * wl.k * 4.0,
        # attention: S = q.c (d_qk) and O = p.v (d_v) per (selected pair, head)
        "attn_flops": 2.0 * selected * wl.H * (wl.D + wl.Dv),
        "attn_bytes": selected * wl.D * 2.0 + rows * wl.H * (wl.D + wl.Dv) * 2.0,
    }


# ------------------------------------------------------------------------------------ our arm

class Runner:
    """Inputs resident on the device, outputs and workspace preallocated."""

    def __init__(self, wl, seed, device="cuda", low_memory=False):
        import sparse_attention_19_b200 as dsa
        self.dsa = dsa
        self.wl = wl
        self.device = device
        chunk = wl.chunk if wl.chunk else wl.Lq
        self.chunks = []
        keys = make_key_side(wl, device, seed)
        self.keys = keys
        n_chunks = wl.Lq // chunk
        for c in range(n_chunks):
            if wl.chunk:
                qs = make_query_side(wl, device, seed, chunk_index=c, Lq=chunk)
                q_offset = wl.q_offset + c * chunk
            else:
                qs = make_query_side(wl, device, seed)
                q_offset = wl.q_offset
            self.chunks.append((q_offset, qs))
        self.chunk_len = chunk
        B, H, Dv, k = wl.B, wl.H, wl.Dv, wl.k
        self.indices = torch.empty(B, wl.Lq, k, dtype=torch.int32, device=device)
        self.out = torch.empty(B, wl.Lq, H, Dv, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(B, wl.Lq, H, dtype=torch.float32, device=device)
        ws = 0
        for q_offset, qs in self.chunks:
            ia = dsa._indexer_args(qs["q_I"], qs["q_scale"], qs["w"], keys["k_I"][:, : q_offset + chunk],
                                   keys["k_scale"][:, : q_offset + chunk], q_offset)
            op = dsa.OP_FORWARD_LOWMEM if low_memory else dsa.OP_FORWARD
            ws = max(ws, dsa.workspace_size_args(op, ia, k, H, Dv))
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.low_memory = low_memory
        # per forward call: the indexer and the top-k (one fused launch in low-memory
        # mode), the attention, and its split-k merge when rows are split
        self.launches_per_call = (2 if low_memory else 3) + \
            (1 if dsa.workspace_size(dsa.OP_SPARSE_ATTN, B, chunk, wl.Lk, k, H, Dv) else 0)
        self.work = [work_model(wl, chunk, q0) for q0, _ in self.chunks]

    def step(self, stream, events=None):
        self.forward_into(stream, self.chunks, self.keys, self.indices, self.out, self.lse, events)

    def forward_into(self, stream, chunks, keys, indices, out, lse, events=None):
        """One forward pass over the given device buffers (the runner's own, or another set)."""
        wl, c = self.wl, self.chunk_len
        for n, (q_offset, qs) in enumerate(chunks):
            Lk = q_offset + c
            sl = slice(n * c, (n + 1) * c) if wl.chunk else slice(None)
            k_I = keys["k_I"][:, :Lk] if wl.chunk else keys["k_I"]
            k_scale = keys["k_scale"][:, :Lk] if wl.chunk else keys["k_scale"]
            kv = keys["kv"][:, :Lk] if wl.chunk else keys["kv"]
            if wl.chunk:   # a chunk's key side is a prefix of the whole sequence (contiguous when B == 1)
                assert wl.B == 1
            self.dsa.forward(qs["q_I"], qs["q_scale"], qs["w"], k_I.contiguous() if wl.B > 1 else k_I,
                             k_scale, qs["q"], kv, wl.k, wl.Dv, wl.scale, q_offset,
                             indices=indices[:, sl], out=out[:, sl], lse=lse[:, sl],
                             workspace=self.ws, stream=stream, low_memory=self.low_memory,
                             stage_events=None if events is None else events[n])

    def totals(self):
        tot = {}
        for w in self.work:
            for k, v in w.items():
                tot[k] = tot.get(k, 0) + v
        return tot


def time_runner(runner, steps, warmup, world, sample_clocks, local):
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        runner.step(stream)
    torch.cuda.synchronize()
    nchunks = len(runner.chunks)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nchunks)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if sample_clocks else None
    if sampler:
        sampler.__enter__()
        time.sleep(0.3)
    start.record(stream)
    for s in range(steps):
        runner.step(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.__exit__()
    barrier(world)
    total_ms = start.elapsed_time(end)
    # The stage breakdown comes from a second pass over the same number of steps
    # with CUDA events recorded between the kernels (events between launches add a
    # few microseconds per step, so they stay out of the timed pass above).
    for s in range(steps):
        runner.step(stream, ev[s])
    torch.cuda.synchronize()
    barrier(world)
    # spans: [0] indexer (with the top-k when fused), [1] top-k (0 when fused),
    # [2] attention + split-k merge
    stage_ms = [0.0, 0.0, 0.0]
    for s in range(steps):
        for c in range(nchunks):
            e = ev[s][c]
            for i in range(3):
                stage_ms[i] += e[i].elapsed_time(e[i + 1])
    stage_ms = [x / steps for x in stage_ms]
    return total_ms / steps, stage_ms, (sampler.summary() if sampler else None)


def roofline_stages(wl, runner, stage_ms, peaks, peak_src):
    tot = runner.totals()
    if "fp8_tflops_sustained" in peaks:
        fp8_sust = peaks["fp8_tflops_sustained"]
        fp8_note = "measured sustained fp8 in this run (" + peaks["fp8_method"] + ")"
    else:
        fp8_sust = 2.0 * peaks["bf16_tflops_sustained"]
        fp8_note = f"fp8 = 2 x {peak_src} sustained bf16 (nominal fp8:bf16 ratio)"
    decode = wl.Lq == 1
    calls = len(runner.chunks)
    out = {}
    # indexer: FP8 contraction for prefill; streams the key cache for decode
    if decode:
        out["indexer"] = dict(bound="hbm", achieved=tot["indexer_bytes"] / (stage_ms[0] * 1e-3) / 1e9,
                              peak=peaks["hbm_gbs"], unit="GB/s", algorithmic=tot["indexer_bytes"] / calls)
    else:
        out["indexer"] = dict(bound="tensor", achieved=tot["indexer_flops"] / (stage_ms[0] * 1e-3) / 1e12,
                              peak=fp8_sust, unit="TFLOP/s", algorithmic=tot["indexer_flops"] / calls,
                              peak_note=fp8_note)
    if runner.low_memory:
        # the selection runs inside the indexer kernel: no top-k launch to time (the
        # span between its events holds no kernel), and the indexer's span covers both
        out["indexer"]["note"] = "indexer with the top-k selection fused into its epilogue"
    elif stage_ms[1] > 0:
        # top-k: a streaming selection over the causal scores
        out["topk"] = dict(bound="hbm", achieved=tot["topk_bytes"] / (stage_ms[1] * 1e-3) / 1e9,
                           peak=peaks["hbm_gbs"], unit="GB/s", algorithmic=tot["topk_bytes"] / calls)
    if decode:
        out["sparse_attn"] = dict(bound="hbm", achieved=tot["attn_bytes"] / (stage_ms[2] * 1e-3) / 1e9,
                                  peak=peaks["hbm_gbs"], unit="GB/s", algorithmic=tot["attn_bytes"] / calls,
                                  tflops=tot["attn_flops"] / (stage_ms[2] * 1e-3) / 1e12)
    else:
        out["sparse_attn"] = dict(bound="tensor", achieved=tot["attn_flops"] / (stage_ms[2] * 1e-3) / 1e12,
                                  peak=peaks["bf16_tflops_sustained"], unit="TFLOP/s",
                                  algorithmic=tot["attn_flops"] / calls)
    total = sum(stage_ms)
    for name, ms in (("indexer", stage_ms[0]), ("topk", stage_ms[1]), ("sparse_attn", stage_ms[2])):
        if name not in out:
            continue
        d = out[name]
        d["ms_per_step"] = ms
        d["frac"] = d["achieved"] / d["peak"]
        d["launches_per_step"] = calls
        d["share"] = ms / total if total > 0 else None
    return out


def topk_kernel_name(wl, chunk):
    """Which top-k kernel dsa_topk launches for these rows (the library's dispatch rule)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows = wl.B * chunk
    nmax = min(wl.q_offset + wl.Lq, wl.Lk) if not wl.chunk else wl.Lk
    if rows * 4 <= 2 * sms and nmax > 16384:
        return "topk_cluster_kernel"
    return "topk_warp_kernel" if rows >= 16 * sms else "topk_kernel"


def traffic_from_profiles(kernel_name, workload):
    """ncu DRAM bytes per launch recorded under profiles/ for this kernel + workload, if current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
        return d.get(workload, {}).get(kernel_name)
    except Exception:
        return None


def measure_e2e(wl, runner, steps, warmup, world):
    """Public API with pinned host buffers: every step copies its inputs host -> device
    and its outputs (indices, out, lse) device -> host inside the timed region.

    Steps are pipelined the way a caller of the API would run them: two device
    buffer sets, the input copies on one stream, the forward on another, the output
    copies on a third, so step i+1's inputs and step i-1's outputs cross PCIe while
    step i's kernels run.  The timed region starts before the first input copy and
    ends after the last output copy.
    """
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    host_in = [{k: v.cpu().pin_memory() for k, v in qs.items()} for _, qs in runner.chunks]
    host_keys = {k: v.cpu().pin_memory() for k, v in runner.keys.items()}
    own = {"chunks": runner.chunks, "keys": runner.keys, "indices": runner.indices, "out": runner.out,
           "lse": runner.lse}
    other = {"chunks": [(q0, {k: torch.empty_like(v) for k, v in qs.items()}) for q0, qs in runner.chunks],
             "keys": {k: torch.empty_like(v) for k, v in runner.keys.items()},
             "indices": torch.empty_like(runner.indices), "out": torch.empty_like(runner.out),
             "lse": torch.empty_like(runner.lse)}
    slots = [own, other]
    host_out = [{f: torch.empty(getattr(runner, f).shape, dtype=getattr(runner, f).dtype).pin_memory()
                 for f in ("indices", "out", "lse")} for _ in range(2)]
    bi = sum(v.numel() * v.element_size() for v in host_keys.values())
    bi += sum(v.numel() * v.element_size() for d in host_in for v in d.values())
    bo = sum(t.numel() * t.element_size() for t in host_out[0].values())

    def run(n_steps, start_event):
        comp_done, out_done = [], []
        s_in.wait_event(start_event)
        for i in range(n_steps):
            sl, ho = slots[i % 2], host_out[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])           # the slot's inputs are free
                for k, v in host_keys.items():
                    sl["keys"][k].copy_(v, non_blocking=True)
                for (_, qs), hd in zip(sl["chunks"], host_in):
                    for k, v in hd.items():
                        qs[k].copy_(v, non_blocking=True)
                in_done = torch.cuda.Event()
                in_done.record(s_in)
            comp.wait_event(in_done)
            if i >= 2:
                comp.wait_event(out_done[i - 2])                # the slot's outputs were read back
            runner.forward_into(comp, sl["chunks"], sl["keys"], sl["indices"], sl["out"], sl["lse"])
            ev = torch.cuda.Event()
            ev.record(comp)
            comp_done.append(ev)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev)
                for f in ("indices", "out", "lse"):
                    ho[f].copy_(sl[f], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(s_out)
                out_done.append(ev_o)
        comp.wait_event(out_done[-1])

    first = torch.cuda.Event()
    first.record(comp)
    run(warmup, first)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    run(steps, s)
    e.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e) / steps, world)
    del other, slots
    return ms, bi, bo


def time_dense_vs_gather(steps, warmup, world, peaks, seed=0):
    """Short-sequence leg (L = k = 2048): the forward pass in its dense mode (keys
    0..t read as contiguous tiles, index lists written by the attention kernel)
    beside the gather path on the same input (dsa_sparse_attn over explicit index
    lists 0..t, which gathers every key row through TMA gather4)."""
    import sparse_attention_19_b200 as dsa
    wl = WORKLOADS["prefill_2k"]
    inp = make_inputs(wl, "cuda", seed)
    stream = torch.cuda.current_stream()
    idx = torch.empty(wl.B, wl.Lq, wl.k, dtype=torch.int32, device="cuda")
    out = torch.empty(wl.B, wl.Lq, wl.H, wl.Dv, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.B, wl.Lq, wl.H, dtype=torch.float32, device="cuda")
    ws_f = torch.empty(max(256, dsa.workspace_size(dsa.OP_FORWARD, wl.B, wl.Lq, wl.Lk, wl.k, wl.H, wl.Dv)),
                       dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(max(256, dsa.workspace_size(dsa.OP_SPARSE_ATTN, wl.B, wl.Lq, wl.Lk, wl.k, wl.H, wl.Dv)),
                       dtype=torch.uint8, device="cuda")
    g_idx = torch.empty_like(idx)
    g_out, g_lse = torch.empty_like(out), torch.empty_like(lse)

    def dense():
        dsa.forward(inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], inp["q"], inp["kv"], wl.k,
                    wl.Dv, wl.scale, 0, indices=idx, out=out, lse=lse, workspace=ws_f, stream=stream)

    dense()
    torch.cuda.synchronize()
    g_idx.copy_(idx)                                   # 0..t, -1 padded

    def gather():
        dsa.sparse_attn(inp["q"], inp["kv"], g_idx, wl.Dv, wl.scale, out=g_out, lse=g_lse, workspace=ws_a,
                        stream=stream)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        barrier(world)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(steps):
            fn()
        e.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(s.elapsed_time(e) / steps, world)

    ms_d, ms_g = timed(dense), timed(gather)
    tot = work_model(wl)
    res = {}
    for name, ms in (("dense", ms_d), ("gather", ms_g)):
        tf = tot["attn_flops"] / (ms * 1e-3) / 1e12
        res[name] = {"value": tot["rows"] * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
                     "attn_tflops": tf, "frac": tf / peaks["bf16_tflops"],
                     "peak": peaks["bf16_tflops"], "peak_note": "burst bf16 (a kernel timed on its own)"}
    res["speedup_dense_over_gather"] = ms_g / ms_d
    res["same_result"] = bool(torch.equal(out, g_out) and torch.equal(lse, g_lse))
    res["workload"] = wl.name
    res["steps"] = steps
    return res


def selected_scores(runner):
    """One more forward pass of the headline step that also returns the indexer
    score of every selected position (fp32 [B, Lq, k]), for the loss leg."""
    wl = runner.wl
    sel = torch.empty(wl.B, wl.Lq, wl.k, dtype=torch.float32, device=runner.device)
    q_offset, qs = runner.chunks[0]
    runner.dsa.forward(qs["q_I"], qs["q_scale"], qs["w"], runner.keys["k_I"], runner.keys["k_scale"], qs["q"],
                       runner.keys["kv"], wl.k, wl.Dv, wl.scale, q_offset, indices=runner.indices, out=runner.out,
                       lse=runner.lse, workspace=runner.ws, sel_scores=sel)
    torch.cuda.synchronize()
    return sel


def time_indexer_kl(wl, runner, steps, warmup, world, peaks, peak_src, sel):
    """The indexer's training loss (forward) on the step's own outputs: its selection,
    the selected positions' scores and its lse.  One launch per call."""
    dsa = runner.dsa
    _, qs = runner.chunks[0]
    B, Lq, k = wl.B, wl.Lq, wl.k
    target = torch.empty(B, Lq, k, dtype=torch.float32, device=runner.device)
    kl = torch.empty(B, Lq, dtype=torch.float32, device=runner.device)
    stream = torch.cuda.current_stream()

    def call():
        dsa.indexer_kl_loss_selected(qs["q"], runner.keys["kv"], runner.indices, runner.lse, sel, wl.Dv, wl.scale,
                                     target=target, kl=kl, stream=stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        call()
    e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e) / steps, world)
    tot = runner.totals()
    # S = q . c over every (selected pair, head); gathered latent rows as the bytes
    flops = 2.0 * tot["selected_pairs"] * wl.H * wl.D
    achieved = flops / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"workload": wl.name, "value": tot["rows"] * world / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": steps, "warmup": warmup, "gpu_launches": steps,
            "roofline": {"kernel": "indexer_kl_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "per_launch_algorithmic": flops,
                         "peak_source": f"{peak_src} burst bf16 (MEASURED_PEAKS.json)",
                         "gathered_gb": tot["selected_pairs"] * wl.D * 2 / 1e9,
                         "traffic": traffic_from_profiles("indexer_kl_kernel", wl.name)},
            "kl_mean": float(kl.mean())}


def cpu_baseline_kl(wl, runner, sel_scores, budget_s=8.0):
    """The oracle's indexer loss on rows spread evenly over the workload (host cores),
    on the step's own selection, selected scores and lse inputs."""
    import oracle
    cores = oracle.num_threads()
    _, qs = runner.chunks[0]
    B, Lq, Lk, k = wl.B, wl.Lq, wl.Lk, wl.k
    kv = runner.keys["kv"].cpu().view(torch.int16).numpy().view(np.uint16)

    def sample(n):
        rows = np.unique(np.linspace(0, B * Lq - 1, n).astype(np.int64))
        sel = torch.as_tensor(rows, device=runner.device)
        q = qs["q"].reshape(B * Lq, wl.H, wl.D)[sel].cpu().view(torch.int16).numpy().view(np.uint16)
        idx = runner.indices.reshape(B * Lq, k)[sel].cpu().numpy()
        # the oracle takes a row of scores over all positions; only the selected ones are read
        ss = sel_scores.reshape(B * Lq, k)[sel].double().cpu().numpy()
        sc = np.zeros((len(rows), Lk))
        for j in range(len(rows)):
            ok = idx[j] >= 0
            sc[j, idx[j][ok]] = ss[j][ok]
        t0 = time.perf_counter()
        oracle.indexer_kl(rows // Lq, q, kv, idx, sc, wl.scale)
        return len(rows), time.perf_counter() - t0

    n, dt = sample(max(cores, 4))
    n_target = int(min(16 * cores, max(n, n * budget_s / max(dt, 1e-3))))
    if n_target > n * 1.5:
        n, dt = sample(n_target)
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} query rows spread evenly over the {wl.name} workload (the loss of each row "
                      f"over its selected positions), {dt:.1f} s on {cores} threads"}


# ------------------------------------------------------------------------------------ CPU oracle

def oracle_sample(wl, inp_dev_or_host, n_rows, seed=0):
    """Time the oracle on n_rows rows spread evenly over the workload (one chunk for chunked)."""
    import oracle
    rng = np.random.default_rng(seed)
    total = wl.B * wl.Lq
    rows = np.unique(np.linspace(0, total - 1, n_rows).astype(np.int64))
    r = oracle.rows_from_inputs(inp_dev_or_host, rows, wl.Lq, wl.q_offset)
    b_used = np.unique(r["row_b"])
    keys = {
        "k_I": inp_dev_or_host["k_I"][torch.as_tensor(b_used)].cpu().numpy(),
        "k_scale": inp_dev_or_host["k_scale"][torch.as_tensor(b_used)].cpu().numpy(),
        "kv": inp_dev_or_host["kv"][torch.as_tensor(b_used)].cpu().view(torch.int16).numpy().view(np.uint16),
    }
    row_b = np.searchsorted(b_used, r["row_b"])
    t0 = time.perf_counter()
    oracle.dsa_forward(row_b, r["row_t"], r["q_I"], r["q_scale"], r["w"], keys["k_I"], keys["k_scale"], r["q"],
                       keys["kv"], wl.k, wl.scale, wl.Dv)
    return len(rows), time.perf_counter() - t0


def cpu_baseline(wl, inp, budget_s=15.0):
    import oracle
    cores = oracle.num_threads()
    n0 = max(cores, 4)
    n, dt = oracle_sample(wl, inp, n0)
    n_target = int(min(4 * n0 * 64, max(n, n * budget_s / max(dt, 1e-3))))
    if n_target > n * 1.5:
        n, dt = oracle_sample(wl, inp, n_target, seed=1)
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} query rows spread evenly over the {wl.name} workload "
                      f"(all of their indexer pairs, top-k and attention), {dt:.1f} s on {cores} threads"}


def _oracle_inputs(wl, seed):
    """Inputs for the oracle arm: generated on the GPU when there is one (only the
    sampled rows and the key side are copied to the host), else on the host."""
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_key_side(wl, dev, seed)
    if wl.chunk:   # the last chunk's queries stand for the workload
        c = wl.Lq // wl.chunk - 1
        inp.update(make_query_side(wl, dev, seed, chunk_index=c, Lq=wl.chunk))
        return inp, wl.with_(Lq=wl.chunk, q_offset=c * wl.chunk)
    inp.update(make_query_side(wl, dev, seed))
    return inp, wl


def run_reference(args, rank, world):
    """The oracle as the reference arm (host cores), rank 0 only."""
    if rank != 0:
        return
    import oracle
    wl = WORKLOADS[args.workload]
    inp, wl_eff = _oracle_inputs(wl, args.seed)
    cores = oracle.num_threads()
    n_rows = max(2 * cores, 8)
    for _ in range(args.warmup):
        oracle_sample(wl_eff, inp, max(cores // 2, 1))
    total_rows, total_s = 0, 0.0
    for s in range(args.steps):
        n, dt = oracle_sample(wl_eff, inp, n_rows, seed=s)
        total_rows += n
        total_s += dt
    value = total_rows / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {n_rows} query rows spread evenly over {wl_eff.name} "
                                   f"(Lq={wl_eff.Lq}, q_offset={wl_eff.q_offset})"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl):
    l2_note = "inputs larger than L2 (q alone is %.1f GB)" % (wl.B * wl.Lq * wl.H * wl.D * 2 / 1e9)
    return {"workload": wl.name, "B": wl.B, "Lq": wl.Lq, "Lk": wl.Lk, "q_offset": wl.q_offset,
            "chunk": wl.chunk or None, "k": wl.k, "H_I": wl.H_I, "d_I": wl.d_I, "H": wl.H, "d_qk": wl.D,
            "d_v": wl.Dv, "indexer": "fp8 e4m3, per-token fp32 scales", "attention": "bf16, fp32 accumulate",
            "l2": l2_note, "parallelism": "independent problem per GPU"}


# ------------------------------------------------------------------------------------ main

def run_indexer_topk_only(args, world):
    """The fused indexer + top-k alone on the chosen workload (one call per step and
    chunk, inputs resident): a small, self-contained command for profilers."""
    import sparse_attention_19_b200 as dsa
    wl = WORKLOADS[args.workload]
    chunk = wl.chunk or wl.Lq
    keys = make_key_side(wl, "cuda", args.seed)
    keys.pop("kv")
    calls = []
    for c in range(wl.Lq // chunk):
        qs = make_query_side(wl, "cuda", args.seed, chunk_index=c if wl.chunk else -1, Lq=chunk)
        qs.pop("q")
        q0 = wl.q_offset + c * chunk
        L = q0 + chunk if wl.chunk else wl.Lk
        calls.append((q0, qs, keys["k_I"][:, :L], keys["k_scale"][:, :L]))
    torch.cuda.empty_cache()
    idx = torch.empty(wl.B, chunk, wl.k, dtype=torch.int32, device="cuda")
    ws = 0
    for q0, qs, kI, ks in calls:
        ws = max(ws, dsa.workspace_size_args(dsa.OP_INDEXER_TOPK,
                                             dsa._indexer_args(qs["q_I"], qs["q_scale"], qs["w"], kI, ks, q0), wl.k))
    ws = torch.empty(max(ws, 256), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        for q0, qs, kI, ks in calls:
            dsa.indexer_topk(qs["q_I"], qs["q_scale"], qs["w"], kI, ks, wl.k, q0, indices=idx, want_scores=False,
                             workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / args.steps, world)
    tot = work_model(wl)
    print(json.dumps({"stage": "indexer_topk", "workload": wl.name, "ms_per_step": ms, "launches_per_step": len(calls),
                      "tflops": tot["indexer_flops"] / (ms * 1e-3) / 1e12,
                      "gbs": tot["indexer_bytes"] / (ms * 1e-3) / 1e9,
                      "allocated_gb": torch.cuda.memory_allocated() / 1e9}), flush=True)
    assert dsa.device_status() == 0


def main():
    args = parse()
    rank, local, world = dist_init(args)
    if args.stage == "indexer_topk" and args.impl == "ours":
        run_indexer_topk_only(args, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    import sparse_attention_19_b200 as dsa
    peaks, peak_src = load_peaks()
    fp8 = None
    if not args.no_fp8_peak:
        fp8 = measure_fp8_peak()
        peaks["fp8_tflops_sustained"] = fp8["fp8_tflops_sustained"]
        peaks["fp8_method"] = fp8["method"]
    wl = WORKLOADS[args.workload]
    runner = Runner(wl, seed=args.seed + rank)
    ms, stage_ms, clocks = time_runner(runner, args.steps, args.warmup, world, rank == 0, local)
    ms_max = max_over_ranks(ms, world)
    tot = runner.totals()
    tokens = tot["rows"] * world
    value = tokens / (ms_max * 1e-3)
    stages = roofline_stages(wl, runner, stage_ms, peaks, peak_src)
    dom = max((n for n in ("indexer", "topk", "sparse_attn") if n in stages),
              key=lambda n: stages[n]["ms_per_step"])
    d = stages[dom]
    kernel_names = {"indexer": "indexer_kernel", "topk": topk_kernel_name(wl, runner.chunk_len),
                    "sparse_attn": "sparse_attn_kernel"}
    roof = {"kernel": kernel_names[dom], "bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"],
            "unit": d["unit"], "frac": d["frac"],
            "traffic": traffic_from_profiles(kernel_names[dom], wl.name),
            "per_launch_algorithmic": d["algorithmic"], "peak_source": f"{peak_src} (MEASURED_PEAKS.json)"}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8+bf16 (fp32 accumulate)", "data": "synthetic",
        "config": config_of(wl),
        "roofline": roof,
        "stages": {k: {kk: (round(vv, 6) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                   for k, v in stages.items()},
        "selection": "staged: the indexer writes the causal scores, a top-k kernel selects",
        "stage_times": "a second pass of the same steps with CUDA events between the kernels; "
                       "the timed pass records none",
        "gpu_launches": runner.launches_per_call * len(runner.chunks) * args.steps,
        "clocks": clocks,
        "peaks": {"source": f"{peak_src} (MEASURED_PEAKS.json)", "hbm_gbs": peaks["hbm_gbs"],
                  "bf16_tflops": peaks["bf16_tflops"], "bf16_tflops_sustained": peaks["bf16_tflops_sustained"],
                  "fp8": fp8},
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        q_offset0, qs0 = runner.chunks[-1]
        inp = dict(runner.keys, **qs0)
        wl_cpu = wl.with_(Lq=runner.chunk_len, q_offset=q_offset0) if wl.chunk else wl
        line["cpu_baseline"] = cpu_baseline(wl_cpu, inp)
    if not args.no_e2e:
        e_ms, bi, bo = measure_e2e(wl, runner, max(3, args.steps), 1, world)
        line["e2e"] = {"value": tokens / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": bi,
                       "d2h_bytes_per_step": bo, "ms_per_step": e_ms}
    extra = {}
    if (not args.no_extra or args.loss) and not wl.chunk and len(runner.chunks) == 1:
        sel = selected_scores(runner)
        kl_line = time_indexer_kl(wl, runner, max(3, args.steps // 2), args.warmup, world, peaks, peak_src, sel)
        if rank == 0 and world == 1 and not args.no_cpu:
            kl_line["cpu_baseline"] = cpu_baseline_kl(wl, runner, sel)
        extra["indexer_kl_loss"] = kl_line
        del sel
        line["workloads"] = extra
    if not args.no_extra and not wl.chunk:
        # the same forward with the selection fused into the indexer (no score matrix)
        del runner
        torch.cuda.empty_cache()
        runner = Runner(wl, seed=args.seed + rank, low_memory=True)
        steps3 = max(3, args.steps // 4)
        ms3, st3, _ = time_runner(runner, steps3, 3, world, False, local)
        ms3 = max_over_ranks(ms3, world)
        s3 = roofline_stages(wl, runner, st3, peaks, peak_src)
        extra["fused_selection"] = {
            "value": runner.totals()["rows"] * world / (ms3 * 1e-3), "unit": "tokens/s", "ms_per_step": ms3,
            "steps": steps3, "warmup": 3, "workspace_bytes": runner.ws.numel(),
            "stages": {k: {kk: (round(vv, 6) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                       for k, v in s3.items()}}
        line["workloads"] = extra
    if not args.no_extra:
        extra["prefill_2k_dense_vs_gather"] = time_dense_vs_gather(max(5, args.steps), args.warmup, world, peaks)
        for name in ("decode_128k", "prefill_128k"):
            if name == wl.name:
                continue
            del runner
            torch.cuda.empty_cache()
            w2 = WORKLOADS[name]
            runner = Runner(w2, seed=args.seed + rank)
            steps2 = max(3, args.steps // (4 if w2.chunk else 1))
            ms2, st2, _ = time_runner(runner, steps2, 3, world, False, local)
            ms2 = max_over_ranks(ms2, world)
            t2 = runner.totals()
            s2 = roofline_stages(w2, runner, st2, peaks, peak_src)
            extra[name] = {"value": t2["rows"] * world / (ms2 * 1e-3), "unit": "tokens/s", "ms_per_step": ms2,
                           "steps": steps2, "warmup": 3,
                           "stages": {k: {kk: (round(vv, 6) if isinstance(vv, float) else vv)
                                          for kk, vv in v.items()} for k, v in s2.items()}}
        del runner
        torch.cuda.empty_cache()
        line["workloads"] = extra
    assert dsa.device_status() == 0, "a device-side wait gave up during the run"
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
