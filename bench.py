"""Benchmark of one paged-attention batch step on B200.

A step is the whole hot path over one batch of the chosen workload: the
copy-on-write block copies and the cache write of this step's new tokens, then
paged decode (split contexts merged by log-sum-exp) and, for the mixed
workload, chunked prefill.  Default workload: the 70B-like GQA long-context
decode batch (128 sequences, 64 q heads / 8 KV heads, head_dim 128, block 16,
contexts log-uniform in [1024, 32768], about 4.8 GB of K/V per step).

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead.  Under torchrun each rank runs its
own batch (independent sequences, no collective on the data path: weak scaling)
and the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

METRIC = "paged decode tokens/s & KV-read GB/s (% of B200 HBM peak) per batch step"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024  # B200 L2


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(workload: str, rank: int):
    """Seed of rank's batch: rank 0 runs the named workload itself, every other
    rank an independent batch of the same shape (weak scaling)."""
    return None if rank == 0 else synth.CONFIGS[workload]().seed + 100 * rank


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings (the job is as slow as its slowest
    rank).  Without a process group, the values themselves."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


class ClockSampler:
    """SM clock, power and throttle-reason samples while the benchmark runs.

    Reads NVML (read-only queries) every ``interval_s`` from a background
    thread, with host timestamps, so even a timed region of a few milliseconds
    gets samples; ``mark_timed(start, end)`` brackets the timed region and the
    record reports its samples (and those of the whole window for context).
    Falls back to ``nvidia-smi -lms 100`` when NVML cannot be used."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_s: float = 0.002):
        self.idx = device_index
        self.interval = interval_s
        self.samples = []  # (host time, sm MHz, max sm MHz, reasons bitmask, watts)
        self.window = None
        self.thread = None
        self.proc = None
        self.stop_flag = False
        self.source = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return self._start_smi()
        self.source = "nvml"

        def run():
            while not self.stop_flag:
                try:
                    self.samples.append((time.perf_counter(),
                                         pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         smax,
                                         pynvml.nvmlDeviceGetCurrentClocksEventReasons(h),
                                         pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception:
                    pass
                time.sleep(self.interval)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_timed(self, t_start, t_end):
        self.window = (t_start, t_end)

    def _summary(self, rows):
        if not rows:
            return None
        mhz = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n, bit in self.REASONS if r[3] & bit})
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz),
                "sm_max_mhz": max(r[2] for r in rows), "samples": len(rows),
                "reasons": reasons,
                "power_w_median": round(statistics.median(r[4] for r in rows), 1)}

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            rows = list(self.samples)
            timed = rows
            if self.window:
                timed = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
            res = self._summary(timed) or self._summary(rows)
            if res is None:
                return None
            res.update({"source": "nvml", "interval_ms": self.interval * 1e3,
                        "window": "timed region" if timed else "whole run (no sample fell "
                                                                 "inside the timed region)",
                        "whole_run": self._summary(rows)})
            return res
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        mhz, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                mhz.append(float(parts[0]))
                maxes.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes),
                "samples": len(mhz), "reasons": sorted(reasons), "source": "nvidia-smi",
                "window": "warm-up, timed region and e2e leg (100 ms samples)"}


# ----------------------------------------------------------------------------
# the batch step
# ----------------------------------------------------------------------------
class Workload:
    def __init__(self, name, seed, device, kernel=0, partition=0, num_seqs=None):
        import torch
        self.torch = torch
        self.name = name
        kw = {} if seed is None else {"seed": seed}
        if num_seqs:
            kw["batch"] = num_seqs  # a smaller batch of the same shape (profiling)
        self.layout = synth.CONFIGS[name](**kw)
        lay = self.layout
        self.dev = device
        t = synth.fill_device(lay, device)
        self.t = t
        self.dec = lay.decode_rows()
        self.pf = lay.prefill_rows()
        tens = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a), dtype=dt, device=device)
        self.slot_mapping = tens(lay.slot_mapping(), torch.int64)
        self.q_dec = t["q"][tens(synth.token_rows(lay, self.dec), torch.int64)].contiguous() \
            if len(self.dec) else None
        self.tab_dec = tens(lay.block_tables[self.dec], torch.int32)
        self.len_dec = tens(lay.context_lens[self.dec], torch.int32)
        if len(self.pf):
            self.q_pf = t["q"][tens(synth.token_rows(lay, self.pf), torch.int64)].contiguous()
            self.cu_pf = tens(lay.cu_q_lens(self.pf), torch.int32)
            self.tab_pf = tens(lay.block_tables[self.pf], torch.int32)
            self.len_pf = tens(lay.context_lens[self.pf], torch.int32)
            self.max_q_pf = int(lay.q_lens[self.pf].max())
        self.out_dec = torch.empty_like(self.q_dec) if self.q_dec is not None else None
        self.out_pf = torch.empty_like(self.q_pf) if len(self.pf) else None
        import paged_kv_cache_454_b200 as pa
        self.pa = pa
        self.kernel = kernel
        self.partition = partition
        if len(self.dec):
            n = pa.pa_decode_workspace_size(len(self.dec), lay.num_q_heads, t["k_pool"],
                                            lay.max_blocks, partition)
            self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        # algorithmic accounting
        self.bytes_dec = synth.decode_kv_bytes(lay) if len(self.dec) else None
        self.flops_pf = synth.prefill_flops(lay) if len(self.pf) else 0
        self.tokens = len(self.dec) + int(lay.q_lens[self.pf].sum()) if len(self.pf) else len(self.dec)

    # one pass of the hot path; `ev` collects per-component events; `io`
    # optionally replaces the step's input / output tensors (same shapes)
    def step(self, stream, ev=None, io=None):
        pa, lay, t = self.pa, self.layout, self.t
        torch = self.torch
        io = io or {}
        get = lambda name, default: io.get(name, default)

        def mark(name):
            if ev is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                ev.setdefault(name, []).append(e)

        mark("start")
        if lay.copy_pairs.size:
            pa.pa_copy_blocks(t["k_pool"], t["v_pool"], lay.copy_pairs, stream=stream)
        mark("copy")
        pa.pa_reshape_and_cache(get("key", t["key"]), get("value", t["value"]), t["k_pool"],
                                t["v_pool"], get("slot_mapping", self.slot_mapping), stream=stream)
        mark("cache")
        if len(self.pf):
            pa.pa_chunked_prefill(get("q_pf", self.q_pf), get("cu_pf", self.cu_pf), self.max_q_pf,
                                  t["k_pool"], t["v_pool"], get("tab_pf", self.tab_pf),
                                  get("len_pf", self.len_pf), lay.scale,
                                  out=get("out_pf", self.out_pf), stream=stream)
        mark("prefill")
        if len(self.dec):
            pa.pa_decode(get("q_dec", self.q_dec), t["k_pool"], t["v_pool"],
                         get("tab_dec", self.tab_dec), get("len_dec", self.len_dec), lay.scale,
                         out=get("out_dec", self.out_dec), workspace=self.ws, kernel=self.kernel,
                         partition_tokens=self.partition, stream=stream)
        mark("decode")

    def launches_per_step(self):
        """Library kernel launches in one step: block copies (480 pairs per
        launch), the cache write, the decode plan and decode kernel (plus the
        merge kernel on the CUDA-core path), the prefill kernel."""
        lay = self.layout
        n = 1  # cache write
        if lay.copy_pairs.size:
            n += -(-len(lay.copy_pairs) // 480)
        if len(self.dec):
            tensor_core = self.kernel == 2 or (
                self.kernel == 0 and lay.head_dim == 128 and lay.group_size <= 16)
            n += 2 if tensor_core else 3
        if len(self.pf):
            n += 1
        return n


def host_manager_timing(w: Workload, steps: int = 100):
    """Host time of the C++ block manager for this batch's decode steps,
    through the Python binding: every step reserves one new token's slot for
    each decode sequence (``pa_kvm_decode_step``) and brings the batch's block
    tables and lengths up to date (``pa_kvm_batch_update``; the full tables are
    built once before).  No device work."""
    from paged_kv_cache_454_b200.kv_manager import KvManager
    lay = w.layout
    if not len(w.dec):
        return None
    lens = lay.context_lens[w.dec].astype(np.int64)
    S = len(lens)
    max_blocks = int(-(-(int(lens.max()) + steps) // lay.block_size))
    blocks = int(sum(-(-(int(x) + steps) // lay.block_size) for x in lens))
    m = KvManager(blocks, lay.block_size, prefix_caching=False)
    ids = np.arange(S, dtype=np.int64)
    for i in range(S):
        m.add_sequence(i, np.zeros(max(int(lens[i]) - 1, 0), np.int32))
    toks = np.zeros(S, np.int32)
    slots = np.empty(S, np.int64)
    out = (np.empty((S, max_blocks), np.int32), np.empty(S, np.int32))
    m.batch(ids, max_blocks, out=out)
    t0 = time.perf_counter()
    for _ in range(steps):
        m.decode_step(ids, toks, slots=slots)
        m.batch_update(ids, out)
    us = (time.perf_counter() - t0) / steps * 1e6
    m.close()
    return {"us_per_step": round(us, 2), "num_seqs": S, "steps": steps,
            "calls": "pa_kvm_decode_step + pa_kvm_batch_update", "threads": 1}


def sampler_timing(w: Workload, stream, reps: int = 50):
    """Device time of the fused sampler (``pa_sample``) for this batch's decode
    rows at two vocabulary sizes (32000, 152064), temperature 0.7, top-k 50,
    top-p 0.9; CUDA events around ``reps`` calls replayed from a CUDA graph
    after warm-up.  Consecutive calls read different logit buffers whose total
    is over twice the L2, so every call streams its logits from HBM."""
    torch = w.torch
    rows = len(w.dec) if len(w.dec) else 1
    res = {}
    g = torch.Generator(device=w.dev)
    g.manual_seed(0)
    for vocab in (32000, 152064):
        nbuf = -(-2 * L2_BYTES // (rows * vocab * 4)) + 1
        xs = [torch.randn(rows, vocab, device=w.dev, generator=g) * 3 for _ in range(nbuf)]
        T = torch.full((rows,), 0.7, device=w.dev)
        K = torch.full((rows,), 50, dtype=torch.int32, device=w.dev)
        P = torch.full((rows,), 0.9, device=w.dev)
        u = torch.rand(rows, device=w.dev, generator=g)
        out = torch.empty(rows, dtype=torch.int32, device=w.dev)
        with torch.cuda.stream(stream):
            for i in range(max(5, nbuf)):
                w.pa.pa_sample(xs[i % nbuf], T, K, P, u, out=out, stream=stream)
        torch.cuda.synchronize()
        # the calls replayed from a CUDA graph, so the host's per-call binding
        # overhead does not leave the GPU idle between them
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(reps):
                w.pa.pa_sample(xs[i % nbuf], T, K, P, u, out=out,
                               stream=torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            graph.replay()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        res[str(vocab)] = round(e0.elapsed_time(e1) / reps * 1e3, 2)
        del graph, xs
    return {"us_per_call": res, "rows": rows, "temperature": 0.7, "top_k": 50, "top_p": 0.9,
            "l2": "rotating logit buffers, over twice the L2 in total",
            "launch": "calls replayed from a CUDA graph",
            "logits_gb_per_s": {k: round(rows * int(k) * 4 / (v * 1e-6) / 1e9, 1)
                                for k, v in res.items()}}


def swap_timing(w: Workload, stream, blocks: int = 512, reps: int = 10):
    """Device time of moving `blocks` whole blocks (K and V, all KV heads) of this
    pool to page-locked host memory and back (``pa_swap_blocks``), as GB/s
    each way; CUDA events around ``reps`` calls after warm-up."""
    torch = w.torch
    kp, vp = w.t["k_pool"], w.t["v_pool"]
    blocks = min(blocks, kp.shape[0])
    kh = torch.empty((blocks,) + tuple(kp.shape[1:]), dtype=kp.dtype).pin_memory()
    vh = torch.empty_like(kh).pin_memory()
    out_pairs = np.stack([np.arange(blocks), np.arange(blocks)], 1).astype(np.int64)
    res = {}
    for name, direction in (("out", 0), ("in", 1)):
        with torch.cuda.stream(stream):
            for _ in range(2):
                w.pa.pa_swap_blocks(kp, vp, kh, vh, out_pairs, direction, stream=stream)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                w.pa.pa_swap_blocks(kp, vp, kh, vh, out_pairs, direction, stream=stream)
            e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = round(2 * kh.numel() * kh.element_size() / (ms * 1e-3) / 1e9, 1)
    return {"gb_per_s": res, "blocks": blocks,
            "bytes_each_way": 2 * kh.numel() * kh.element_size()}


def probe_timing(w: Workload, stream, decode_ms, reps: int = 20):
    """Device time of ``pa_read_probe`` over this batch's decode tables: it reads
    the very K/V pages the decode call reads (whole pages) and computes nothing,
    one CTA per SM.  ``decode_over_probe`` = probe time / decode time, the share
    of the paged layout's attainable read rate the decode call reaches.  CUDA
    events around ``reps`` calls after warm-up; the pages (GBs) exceed L2."""
    torch = w.torch
    if not len(w.dec):
        return None
    lay = w.layout
    kp, vp = w.t["k_pool"], w.t["v_pool"]
    lens = lay.context_lens[w.dec].astype(np.int64)
    pages = int(sum(-(-int(x) // lay.block_size) for x in lens)) * lay.num_kv_heads
    page_bytes = lay.block_size * lay.head_dim * kp.element_size()
    nbytes = 2 * pages * page_bytes
    ctas = torch.cuda.get_device_properties(kp.device).multi_processor_count
    out = torch.empty(ctas, dtype=torch.int64, device=kp.device)
    with torch.cuda.stream(stream):
        for _ in range(3):
            w.pa.pa_read_probe(kp, vp, w.tab_dec, w.len_dec, num_ctas=ctas, out=out, stream=stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            w.pa.pa_read_probe(kp, vp, w.tab_dec, w.len_dec, num_ctas=ctas, out=out, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    return {"gb_per_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "us_per_call": round(ms * 1e3, 2),
            "page_bytes_read": nbytes, "pages": 2 * pages, "ctas": ctas,
            "decode_over_probe": round(ms / decode_ms, 4) if decode_ms else None}


def step_stats(ev, first, last):
    """min / median / p90 over the component pass's steps of the span between
    two marks (ms)."""
    v = sorted(b.elapsed_time(c) for b, c in zip(ev[first], ev[last]))
    if not v:
        return None
    p90 = v[max(0, math.ceil(0.9 * len(v)) - 1)]  # nearest rank
    return {"min": round(v[0], 4), "median": round(statistics.median(v), 4),
            "p90": round(p90, 4)}


def e2e_run(w: Workload, stream, steps, warmup):
    """The same step through the public API with host buffers: every step copies
    its inputs (q, new K/V, slot mapping, block tables, context lengths) from
    pinned host memory and reads its output back to pinned host memory, all
    inside the timed region.  As a serving loop would, the copies run on their
    own streams with double-buffered device tensors, so step i+1's inputs move
    while step i computes and step i's output moves while step i+1 computes.
    The KV pool itself is device-resident state."""
    torch = w.torch
    names, host, proto = [], {}, {}

    def add(name, tensor):
        host[name] = torch.empty(tensor.shape, dtype=tensor.dtype, pin_memory=True)
        host[name].copy_(tensor.cpu())
        proto[name] = tensor
        names.append(name)

    add("key", w.t["key"])
    add("value", w.t["value"])
    add("slot_mapping", w.slot_mapping)
    if len(w.dec):
        add("q_dec", w.q_dec)
        add("tab_dec", w.tab_dec)
        add("len_dec", w.len_dec)
    if len(w.pf):
        add("q_pf", w.q_pf)
        add("cu_pf", w.cu_pf)
        add("tab_pf", w.tab_pf)
        add("len_pf", w.len_pf)
    out_names = [n for n, o in (("out_dec", w.out_dec), ("out_pf", w.out_pf)) if o is not None]
    out_proto = {"out_dec": w.out_dec, "out_pf": w.out_pf}
    bufs = [{n: torch.empty_like(proto[n]) for n in names} for _ in range(2)]
    for b in bufs:
        for n in out_names:
            b[n] = torch.empty_like(out_proto[n])
    host_out = [{n: torch.empty(out_proto[n].shape, dtype=out_proto[n].dtype, pin_memory=True)
                 for n in out_names} for _ in range(2)]
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = sum(out_proto[n].numel() * out_proto[n].element_size() for n in out_names)
    s_in = torch.cuda.Stream(device=w.dev)
    s_out = torch.cuda.Stream(device=w.dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):   # every event recorded once, so the first waits are no-ops
        ev_comp[b].record(stream)
        ev_out[b].record(stream)

    def copy_in(i):
        b = i % 2
        s_in.wait_event(ev_comp[b])          # step i-2 is done reading buffer b
        with torch.cuda.stream(s_in):
            for n in names:
                bufs[b][n].copy_(host[n], non_blocking=True)
        ev_in[b].record(s_in)

    def compute(i):
        b = i % 2
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])         # step i-2's output has left buffer b
        with torch.cuda.stream(stream):
            w.step(stream, io=bufs[b])
        ev_comp[b].record(stream)

    def copy_out(i):
        b = i % 2
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            for n in out_names:
                host_out[b][n].copy_(bufs[b][n], non_blocking=True)
        ev_out[b].record(s_out)

    def run(n):
        copy_in(0)
        for i in range(n):
            if i + 1 < n:
                copy_in(i + 1)
            compute(i)
            copy_out(i)

    run(warmup)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    run(steps)
    stream.wait_event(ev_out[(steps - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return ms, h2d, d2h


# ----------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ----------------------------------------------------------------------------
def oracle_sample_runner(w: Workload):
    """Returns (prepare(rows), run(prepared, groups)).  ``prepare`` takes host
    copies of exactly the device inputs of some decode rows (before any library
    call wrote to the pools); ``run`` (``oracle_step``) times the oracle's copy /
    cache write / decode over the first ``groups`` KV heads of them."""
    torch = w.torch
    lay = w.layout

    def prepare(rows):
        sub, blocks = synth.subset(lay, rows)
        idx = torch.as_tensor(blocks, device=w.dev)
        bits = lambda x: x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        kp = bits(w.t["k_pool"].index_select(0, idx))
        vp = bits(w.t["v_pool"].index_select(0, idx))
        tok = torch.as_tensor(synth.token_rows(lay, rows), device=w.dev)
        q = bits(w.t["q"].index_select(0, tok))
        key = bits(w.t["key"].index_select(0, tok))
        val = bits(w.t["value"].index_select(0, tok))
        return sub, kp, vp, q, key, val

    return prepare, oracle_step


def oracle_step(prepared, groups=None):
    """Seconds the oracle takes for the copy-on-write copies, the cache write and
    the decode of one prepared slice ``(sub_layout, k_pool, v_pool, q, key,
    value)``, restricted to its first ``groups`` KV heads (KV-head groups are
    independent, so this is an exact slice of the work)."""
    import oracle
    sub, kp, vp, q, key, val = prepared
    ng = sub.num_kv_heads if groups is None else groups
    G = sub.group_size
    kp, vp = kp[:, :ng], vp[:, :ng]
    key, val, q = key[:, :ng], val[:, :ng], q[:, : ng * G]
    t0 = time.perf_counter()
    if sub.copy_pairs.size:
        kp, vp = oracle.copy_blocks(kp, vp, sub.copy_pairs)
    kp, vp = oracle.reshape_and_cache(kp, vp, key, val, sub.slot_mapping())
    oracle.decode(q, kp, vp, sub.block_tables, sub.context_lens, sub.scale)
    return time.perf_counter() - t0


def host_oracle_slices(workload: str, rows: int = 4):
    """Host-only inputs for the reference arm: the workload's first ``rows``
    decode sequences, each over a compact pool of exactly its blocks, drawn on
    the host (``synth.fill_host``: the same shapes, value distribution and
    poisons as the device batch, from NumPy's generator).  Neither torch nor the
    CUDA library is touched."""
    lay = synth.CONFIGS[workload]()
    out = []
    for r in list(lay.decode_rows())[:rows]:
        sub, _ = synth.subset(lay, [int(r)])
        h = synth.fill_host(sub)
        out.append((sub, h["k_pool"], h["v_pool"], h["q"], h["key"], h["value"]))
    return lay, out


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(w: Workload, budget_s=15.0, max_rows=None):
    """Oracle decode tokens/s over a bounded sample of the workload's decode rows
    (taken in order until ~budget_s of CPU time)."""
    if not len(w.dec):
        return None
    prepare, run = oracle_sample_runner(w)
    done, secs = 0, 0.0
    rows = list(w.dec)
    while done < len(rows) and secs < budget_s and (max_rows is None or done < max_rows):
        secs += run(prepare([rows[done]]))
        done += 1
    ctx = int(w.layout.context_lens[rows[:done]].sum())
    return {"value": done / secs, "unit": "tokens/s", "cores": blas_threads(),
            "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": f"first {done} of {len(rows)} decode sequences of {w.name} "
                      f"({ctx} context tokens, all {w.layout.num_q_heads} q heads), "
                      f"{secs:.1f} s of NumPy fp64"}


# ----------------------------------------------------------------------------
# main
# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="gqa70b_long", choices=list(synth.CONFIGS))
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tcgen05"])
    ap.add_argument("--partition", type=int, default=0)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="smaller batch of the same workload shape (profiling captures)")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)

    rank, world, local = dist_env()
    if a.impl == "reference":
        return reference_arm(a, rank, world)

    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    peaks, peak_src = load_peaks()

    w = Workload(a.workload, rank_seed(a.workload, rank), dev, kernel={"auto": 0, "simt": 1, "tcgen05": 2}[a.kernel], partition=a.partition,
                 num_seqs=a.num_seqs or None)
    # host copies for the CPU baseline are taken before any kernel touches the pools
    cpu = None
    if rank == 0 and world == 1 and not a.skip_cpu_baseline:
        cpu = cpu_baseline(w, a.cpu_budget)

    stream = torch.cuda.Stream(device=dev)
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(a.warmup):
        w.step(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    # The timed region, in two passes under one clock record.  First the
    # component pass: an event between the calls of each step, so each span
    # is that call's own time (the events keep a call from starting before the
    # previous one ends, i.e. no programmatic overlap of the decode plan with
    # the cache write); the decode roofline is taken from it.  Then the
    # headline pass: whole steps with no events between the calls, as a
    # serving loop runs them.
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    h0 = time.perf_counter()
    ev = {}
    comp_steps = min(a.steps, 50)
    for _ in range(comp_steps):
        w.step(stream, ev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(a.steps):
        w.step(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_timed(h0, time.perf_counter())
    if pg:
        pg.barrier()
    ms = t0.elapsed_time(t1) / a.steps
    comp = {}
    names = ["start", "copy", "cache", "prefill", "decode"]
    for i in range(1, len(names)):
        comp[names[i]] = sum(b.elapsed_time(c) for b, c in zip(ev[names[i - 1]], ev[names[i]])) / comp_steps
    e2e = None
    if not a.skip_e2e:
        e2e_ms, h2d, d2h = e2e_run(w, stream, max(10, a.steps // 4), a.warmup)
    clk = clocks.stop()
    if pg:
        ms, e2e_ms = max_over_ranks([ms, e2e_ms if not a.skip_e2e else 0.0], pg, dev)
    if not a.skip_e2e:
        e2e = {"value": world * w.tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    lay = w.layout
    value = world * w.tokens / (ms * 1e-3)
    # roofline of the dominant kernel
    roof = None
    if len(w.dec) and (comp["decode"] >= comp["prefill"]):
        b = w.bytes_dec
        algo = b["unique"]
        achieved = algo / (comp["decode"] * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": "pa_decode (plan and decode launches)",
                "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peak_src} hbm_gbs",
                "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
                "algorithmic_bytes": algo, "logical_bytes": b["logical"],
                "kernel_ms": round(comp["decode"], 4), "traffic": traffic_for(a.workload, "decode")}
    # the chunked prefill's own roofline (the dominant kernel's when it is the
    # longer part of the step)
    roof_pf = None
    if len(w.pf):
        achieved = w.flops_pf / (comp["prefill"] * 1e-3) / 1e12
        pk = peaks["bf16_tflops_sustained"]
        roof_pf = {"bound": "tensor", "kernel": "pa_chunked_prefill", "achieved": round(achieved, 1),
                   "peak": pk, "unit": "TFLOP/s", "frac": round(achieved / pk, 4),
                   "peak_source": f"{peak_src} bf16_tflops_sustained",
                   "algorithmic_flops": w.flops_pf, "kernel_ms": round(comp["prefill"], 4),
                   "traffic": traffic_for(a.workload, "prefill") if not a.num_seqs else None}
        if roof is None:
            roof = roof_pf
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 K/V/q; shuffled block pool; no dataset)",
        "config": {"workload": a.workload if not a.num_seqs else f"{a.workload} (batch {a.num_seqs})",
                   "num_seqs": lay.num_seqs,
                   "decode_seqs": int(len(w.dec)), "prefill_tokens": int(lay.q_lens[w.pf].sum()) if len(w.pf) else 0,
                   "num_q_heads": lay.num_q_heads, "num_kv_heads": lay.num_kv_heads,
                   "head_dim": lay.head_dim, "block_size": lay.block_size,
                   "context_tokens": int(lay.context_lens.sum()), "pool_blocks": lay.num_blocks,
                   "kernel": a.kernel, "partition_tokens": a.partition or "default",
                   "l2": "inputs larger than L2 (K/V read per step %.2f GB vs 126 MB L2)"
                         % ((w.bytes_dec["kv"] if w.bytes_dec else 0) / 1e9),
                   "parallelism": f"replicas x{world} (independent batches per GPU)"},
        "components_ms": {k: round(v, 4) for k, v in comp.items()},
        "step_ms_stats": step_stats(ev, "start", "decode"),
        "decode_ms_stats": step_stats(ev, "prefill", "decode") if len(w.dec) else None,
        "prefill_ms_stats": step_stats(ev, "cache", "prefill") if len(w.pf) else None,
        "kv_gbs": round(w.bytes_dec["unique"] / (comp["decode"] * 1e-3) / 1e9, 1) if len(w.dec) else None,
        "roofline": roof,
        "roofline_prefill": roof_pf if roof_pf is not roof else None,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": w.launches_per_step() * a.steps,
        "clocks": clk,
        "host_block_manager": host_manager_timing(w) if rank == 0 else None,
        "fused_sampler": sampler_timing(w, stream) if rank == 0 else None,
        "block_swap": swap_timing(w, stream) if rank == 0 else None,
        "read_probe": probe_timing(w, stream, comp["decode"]) if rank == 0 else None,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of a
# kernel from an ncu capture, keyed by (workload, kernel) and the sources the
# kernel was built from (reported as null once those sources change).  The
# decode figures are captures of a smaller batch of the same shape, scaled to
# the full batch by algorithmic bytes: gqa70b_long from 48 sequences
# (1,759,879,168 bytes for 1,755,018,024 algorithmic), llama13b_sampling from
# 64 sequences (558,791,168 for 542,159,500 unique).  The prefill figure is the
# mixed step's prefill part itself (its 8 chunks, with the decode part shrunk
# to 8 sequences: the prefill launch is the same).  The captures are
# summarised in profiles/.
TRAFFIC = {
    ("gqa70b_long", "decode"): {"bytes": 4773729483, "sources": "f7116353621e"},
    ("llama13b_sampling", "decode"): {"bytes": 2174878746, "sources": "f7116353621e"},
    ("mixed_qwen32b", "prefill"): {"bytes": 185013760, "sources": "d5dda8f04e86"},
}


# the sources each path's kernels are built from: decode (plan, tensor-core
# decode) and chunked prefill
KERNEL_SOURCES = {
    "decode": ("decode_plan.cu", "decode_tc.cu", "common.cuh", "tc_common.cuh"),
    "prefill": ("prefill_tc.cu", "common.cuh", "tc_common.cuh"),
}


def kernel_source_digest(kind="decode"):
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "paged_kv_cache_454_b200", "csrc")
    for f in KERNEL_SOURCES[kind]:
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:12]


def traffic_for(workload, kind="decode"):
    rec = TRAFFIC.get((workload, kind))
    if not rec or rec.get("sources") != kernel_source_digest(kind):
        return None
    return rec["bytes"]


def reference_arm(a, rank, world):
    """The CPU oracle as the reference: each step runs the oracle over a bounded
    slice (some KV-head groups of one decode sequence) of the same workload,
    sized so the whole run stays within about two minutes.  Its inputs are drawn
    on the host; this arm imports neither torch nor the CUDA library."""
    if rank != 0:
        return
    lay, prepared = host_oracle_slices(a.workload)
    hkv = lay.num_kv_heads
    probe = max(oracle_step(p, 1) for p in prepared)  # one KV group of the longest sample
    budget = 120.0 / (a.steps + a.warmup)
    groups = int(max(1, min(hkv, budget // max(probe, 1e-6))))
    for i in range(a.warmup):
        oracle_step(prepared[i % len(prepared)], groups)
    secs, toks = 0.0, 0.0
    for i in range(a.steps):
        secs += oracle_step(prepared[i % len(prepared)], groups)
        toks += groups / hkv
    value = toks / secs
    sample = (f"each step: oracle copy/cache-write/decode of {groups} of {hkv} KV-head groups "
              f"(all their q heads) of one decode sequence of {a.workload} (cycling over the "
              f"first {len(prepared)}; inputs drawn on the host with the workload's shapes), "
              f"NumPy fp64; counted as {groups}/{hkv} of a token")
    res = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
           "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
           "ms_per_step": secs / max(1, a.steps) * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": a.workload},
           "cpu_baseline": {"kind": "oracle", "cores": blas_threads(), "host_cpus": os.cpu_count(),
                            "sample": sample, "value": value, "unit": "tokens/s"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
