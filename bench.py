#!/usr/bin/env python3
"""Benchmark of the libattn hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--all] [--no-cpu-baseline]

One JSON line on stdout (rank 0). A step is one call sequence of the
library on one batch of the workload, with inputs resident in HBM:
prefill = one attn_fwd_varlen call; paged decode = attn_sched_metadata +
attn_fwd_paged_kvcache (which runs the split kernel and the combine);
MLA = attn_sched_metadata + mla_fwd_paged / mla_sparse_fwd.

The headline workload is the varlen causal GQA prefill (8 sequences with
lengths uniform in [512, 4096], H_q=32, H_kv=8, D=128, bf16); the other
workloads appear under "workloads" with their own roofline. Timing: CUDA
events on the launch stream around every step, an L2 flush (a 512 MiB write)
between steps, W >= 3 untimed warm-up steps, barrier + synchronize on both
sides, max over ranks. Multi-GPU runs are weak scaling: every rank runs its
own copy of the workload (seed + rank) with no collective on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_online_softmax_fmha_b200 import binding as B  # noqa: E402
from attention_online_softmax_fmha_b200 import workloads as W  # noqa: E402

METRIC = "prefill TFLOP/s & decode KV GB/s on 1 B200; % of tensor/HBM roofline"
HEADLINE = "varlen_causal_gqa"
# Timed beside the headline in a default run, each with its own roofline: the
# decode half of the metric, the other prefill configurations and MLA.
DEFAULT_EXTRA = ["paged_decode", "paged_decode_fp8", "window_sink", "window_sink_fp8",
                 "mla_dense", "mla_sparse", "mla_dense_fp8", "mla_sparse_fp8"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# peaks, clocks, traffic
# ---------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic():
    """Per-kernel DRAM bytes per launch from a committed ncu capture, keyed
    by the kernel and the hash of the sources it was built from."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    with open(p) as f:
        return json.load(f)


# The sources each kernel family is built from: its device code, its
# launch code and the shared device and host helpers.
_FAMILY_SOURCES = {
    "prefill_kernel": ["prefill_sm100.cuh", "prefill_host.cuh"],
    "decode_kernel": ["decode_paged.cuh", "sched.cuh", "combine.cuh", "sched_host.cuh", "api.cu"],
    "mla_kernel": ["mla_sm100.cuh", "sched.cuh", "combine.cuh", "sched_host.cuh", "mla_host.cuh"],
}


def source_hash(kernel: str = None) -> str:
    """Hash of the sources a kernel is built from (all kernel sources when
    `kernel` is None); keys the committed ncu traffic figures."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_online_softmax_fmha_b200", "csrc")
    family = None
    if kernel is not None:
        family = _FAMILY_SOURCES.get(kernel.split("<")[0])
    names = sorted(os.listdir(csrc)) if family is None else sorted(
        family + ["common.cuh", "host.cuh"])
    for name in names:
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout: float):
        t0 = time.perf_counter()
        while self.proc is not None and not self.lines and time.perf_counter() - t0 < timeout:
            time.sleep(0.02)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# workloads: each returns a dict with the device step, the host (e2e) step,
# the algorithmic work and the roofline description
# ---------------------------------------------------------------------------

def _visible_pairs(lq: int, lk: int, causal: bool, wl: int, wr: int) -> int:
    """Visible (query, key) pairs of one sequence and head, summed in closed
    form row by row: row i sees keys [max(0, i+d-wl), min(lk-1, i+d[+wr]))."""
    d = lk - lq
    tot = 0
    for i in range(lq):
        lo = 0 if wl < 0 else max(0, i + d - wl)
        hi = lk - 1
        if causal:
            hi = min(hi, i + d)
        if wr >= 0:
            hi = min(hi, i + d + wr)
        if hi >= lo:
            tot += hi - lo + 1
    return tot


def prefill_workload(name: str, seed: int, device):
    inp = W.build_config(name, seed=seed, device=device)
    D = inp.head_dim
    pairs = sum(_visible_pairs(a, b, inp.causal, inp.window[0], inp.window[1])
                for a, b in zip(inp.seqlens_q, inp.seqlens_k))
    flops = 2.0 * (D + D) * inp.num_heads_q * pairs
    kw = dict(scale=inp.scale, causal=inp.causal, window=inp.window, sink=inp.sink,
              q_descale=inp.q_descale, k_descale=inp.k_descale, v_descale=inp.v_descale,
              mask=inp.mask)
    if inp.varlen:
        kw.update(cu_seqlens_q=inp.cu_seqlens_q, cu_seqlens_k=inp.cu_seqlens_k,
                  max_seqlen_q=max(inp.seqlens_q), max_seqlen_k=max(inp.seqlens_k))
    args, out, lse = B.varlen_args(inp.q, inp.k, inp.v, **kw)
    L = B.lib()
    import ctypes

    def step(stream):
        st = L.attn_fwd_varlen(ctypes.byref(args), stream.cuda_stream)
        if st != B.OK:
            raise B.AttnError("attn_fwd_varlen", st)

    # e2e: pinned host copies of the step's inputs; H2D, the call, D2H of out/lse
    host_in = [t.cpu().pin_memory() for t in (inp.q, inp.k, inp.v)]
    # (FP8 tensors are copied as raw bytes)
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                torch.empty(lse.shape, dtype=lse.dtype).pin_memory()]
    dev_in = [inp.q, inp.k, inp.v]
    small = [t for t in (inp.cu_seqlens_q, inp.cu_seqlens_k, inp.sink, inp.q_descale,
                         inp.k_descale, inp.v_descale) if t is not None]
    if inp.mask is not None:  # the mask's storage (rows padded to 4 floats)
        small.append(inp.mask.as_strided((inp.mask.numel() // inp.mask.shape[-1] *
                                           inp.mask.stride(2),), (1,)))
    host_small = [t.cpu().pin_memory() for t in small]

    def e2e_step(stream):
        for h, d in zip(host_in + host_small, dev_in + small):
            d.copy_(h, non_blocking=True)
        step(stream)
        host_out[0].copy_(out, non_blocking=True)
        host_out[1].copy_(lse, non_blocking=True)

    h2d = sum(t.numel() * t.element_size() for t in host_in + host_small)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    bound = "tensor"
    cfg = {"workload": name, "batch": inp.batch, "seqlens": "uniform[512,4096]" if inp.varlen
           else inp.seqlens_q[0], "num_heads_q": inp.num_heads_q, "num_heads_kv": inp.num_heads_kv,
           "head_dim": D, "causal": inp.causal, "window": list(inp.window),
           "sink": inp.sink is not None, "dtype": inp.dtype, "total_q_tokens": sum(inp.seqlens_q),
           "visible_pairs_per_head": pairs, "additive_mask": inp.mask is not None}
    kernel = f"prefill_kernel<{D},{ {'bf16': 0, 'fp16': 1, 'e4m3': 2, 'e5m2': 3}[inp.dtype] }>"
    return dict(step=step, e2e_step=e2e_step, work=flops / 1e12, unit="TFLOP/s", bound=bound,
                kernel=kernel, launches_per_step=1, h2d=h2d, d2h=d2h, cfg=cfg,
                dtype=inp.dtype, inp=inp, outputs=(out, lse),
                per_unit=f"2*(D_qk+D_v)*H_q FLOP per visible pair, "
                f"{pairs} visible pairs per head")


def paged_workload(name: str, seed: int, device):
    inp = W.build_config(name, seed=seed, device=device)
    D, Hq, Hkv, B_ = inp.head_dim, inp.num_heads_q, inp.num_heads_kv, inp.batch
    sq = inp.q.shape[1]
    import ctypes
    L = B.lib()
    sa = B.sched_args(inp.cache_seqlens, batch=B_, seqlen_q=sq, num_heads_q=Hq,
                      num_heads_kv=Hkv, head_dim_qk=D, head_dim_v=D, page_size=inp.page_size)
    meta = torch.empty(B.sched_metadata_size(sa) // 4, dtype=torch.int32, device=device)
    sa.meta = meta.data_ptr()
    sa.meta_bytes = meta.numel() * 4
    pa, out, lse, ws = B.paged_args(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                    inp.cache_seqlens, scale=inp.scale, causal=inp.causal,
                                    window=inp.window, sink=inp.sink, meta=meta,
                                    q_descale=inp.q_descale, k_descale=inp.k_descale,
                                    v_descale=inp.v_descale)
    # algorithmic bytes: every visible K and V row once per KV head, Q, O, LSE,
    # the used block-table entries and cache_seqlens (and the FP8 descales)
    kv_rows = sum(inp.seqlens)
    pages = sum(-(-x // inp.page_size) for x in inp.seqlens)
    es = inp.k_cache.element_size()
    fp8 = inp.q_descale is not None
    nbytes = (kv_rows * Hkv * 2 * D * es + inp.q.numel() * inp.q.element_size()
              + out.numel() * 2 + lse.numel() * 4 + pages * 4 + B_ * 4
              + (3 * B_ * Hkv * 4 if fp8 else 0))

    def step(stream):
        st = L.attn_sched_metadata(ctypes.byref(sa), stream.cuda_stream)
        if st != B.OK:
            raise B.AttnError("attn_sched_metadata", st)
        st = L.attn_fwd_paged_kvcache(ctypes.byref(pa), stream.cuda_stream)
        if st != B.OK:
            raise B.AttnError("attn_fwd_paged_kvcache", st)

    # e2e: the step's inputs are the new query rows, the block table and the
    # cache lengths (the KV cache is resident state); out and LSE come back.
    small = [inp.q, inp.block_table, inp.cache_seqlens]
    host_small = [t.cpu().pin_memory() for t in small]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                torch.empty(lse.shape, dtype=lse.dtype).pin_memory()]

    def e2e_step(stream):
        for h, d in zip(host_small, small):
            d.copy_(h, non_blocking=True)
        step(stream)
        host_out[0].copy_(out, non_blocking=True)
        host_out[1].copy_(lse, non_blocking=True)

    cfg = {"workload": name, "batch": B_, "seqlen_q": sq, "num_heads_q": Hq,
           "num_heads_kv": Hkv, "head_dim": D, "page_size": inp.page_size,
           "cache_seqlens": "uniform[1024,32768]", "block_table": "seeded permutation",
           "kv_tokens": kv_rows, "dtype": inp.dtype}
    return dict(step=step, e2e_step=e2e_step, work=nbytes / 1e9, unit="GB/s", bound="hbm",
                kernel="decode_kernel<128,%d>" % (2 if fp8 else 0), launches_per_step=3,
                h2d=sum(t.numel() * t.element_size() for t in host_small),
                d2h=sum(t.numel() * t.element_size() for t in host_out), cfg=cfg,
                dtype=inp.dtype, inp=inp, keep=(meta, ws, out, lse), outputs=(out, lse),
                per_unit=f"(D_k + D_v) * {es} B per cached token per KV head + Q/O/LSE/table; "
                f"{nbytes} B per step")


def mla_workload(name: str, seed: int, device):
    inp = W.build_config(name, seed=seed, device=device)
    import ctypes
    L = B.lib()
    sparse = inp.indices is not None
    sq, Hq = inp.q.shape[1], inp.num_heads_q
    topk = inp.topk if sparse else 0
    sa = B.sched_args(inp.cache_seqlens, batch=inp.batch, seqlen_q=sq, num_heads_q=Hq,
                      num_heads_kv=1, head_dim_qk=576, head_dim_v=512, page_size=inp.page_size,
                      mode=B.SCHED_MLA_SPARSE if sparse else B.SCHED_MLA, topk=topk)
    meta = torch.empty(B.sched_metadata_size(sa) // 4, dtype=torch.int32, device=device)
    sa.meta = meta.data_ptr()
    sa.meta_bytes = meta.numel() * 4
    ma, out, lse, ws = B.mla_args(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens,
                                  scale=inp.scale, causal=inp.causal, indices=inp.indices,
                                  meta=meta, q_descale=inp.q_descale, k_descale=inp.k_descale,
                                  v_descale=inp.v_descale)
    fp8 = inp.dtype == "e4m3"
    es = inp.kv_cache.element_size()
    fn = L.mla_sparse_fwd if sparse else L.mla_fwd_paged
    if sparse:
        idx = inp.indices.cpu()
        lens = torch.tensor(inp.seqlens).view(-1, 1, 1, 1)
        pairs_tok = int(((idx >= 0) & (idx < lens)).sum())   # visible keys over all tokens
        kv_rows = pairs_tok
    else:
        pairs_tok = sum(inp.seqlens) * sq
        kv_rows = sum(inp.seqlens)
    flops = 2.0 * (576 + 512) * Hq * pairs_tok
    nbytes = (kv_rows * 576 * es + inp.q.numel() * es + out.numel() * 2 + lse.numel() * 4
              + (3 * inp.batch * 4 if fp8 else 0))

    def step(stream):
        st = L.attn_sched_metadata(ctypes.byref(sa), stream.cuda_stream)
        if st != B.OK:
            raise B.AttnError("attn_sched_metadata", st)
        st = fn(ctypes.byref(ma), stream.cuda_stream)
        if st != B.OK:
            raise B.AttnError(name, st)

    small = [inp.q, inp.block_table, inp.cache_seqlens] + ([inp.indices] if sparse else []) + (
        [inp.q_descale, inp.k_descale, inp.v_descale] if fp8 else [])
    host_small = [t.cpu().pin_memory() for t in small]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                torch.empty(lse.shape, dtype=lse.dtype).pin_memory()]

    def e2e_step(stream):
        for h, d in zip(host_small, small):
            d.copy_(h, non_blocking=True)
        step(stream)
        host_out[0].copy_(out, non_blocking=True)
        host_out[1].copy_(lse, non_blocking=True)

    cfg = {"workload": name, "batch": inp.batch, "seqlen_q": sq, "num_heads_q": Hq,
           "num_heads_kv": 1, "head_dim_qk": 576, "head_dim_v": 512, "page_size": inp.page_size,
           "cache_seqlens": "uniform[4096,65536]", "topk": topk or None, "dtype": inp.dtype,
           "kv_bytes_per_step": nbytes}
    return dict(step=step, e2e_step=e2e_step, work=flops / 1e12, unit="TFLOP/s", bound="tensor",
                kernel=f"mla_kernel<{int(sparse)},{int(fp8)}>", launches_per_step=3,
                h2d=sum(t.numel() * t.element_size() for t in host_small),
                d2h=sum(t.numel() * t.element_size() for t in host_out), cfg=cfg, dtype=inp.dtype,
                inp=inp, keep=(meta, ws, out, lse), outputs=(out, lse), gbytes=nbytes / 1e9,
                per_unit=f"2*(576+512)*H_q FLOP per visible (token, key) pair; "
                f"{pairs_tok} pairs, {nbytes} bytes per step")


WORKLOADS = {
    "tiny_dense_mha": prefill_workload,
    "varlen_causal_gqa": prefill_workload,
    "window_sink": prefill_workload,
    "window_sink_fp8": prefill_workload,
    "window_sink_e5m2": prefill_workload,
    "dense_mask": prefill_workload,
    "paged_decode": paged_workload,
    "paged_decode_small": paged_workload,
    "paged_decode_fp8": paged_workload,
    "mla_dense": mla_workload,
    "mla_sparse": mla_workload,
    "mla_dense_fp8": mla_workload,
    "mla_sparse_fp8": mla_workload,
    "paged_decode_fp8_small": paged_workload,
    "mla_dense_fp8_small": mla_workload,
    "mla_sparse_fp8_small": mla_workload,
    "mla_dense_small": mla_workload,
    "mla_sparse_small": mla_workload,
}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------

def cpu_baseline(name: str, seed: int, budget_s: float = 15.0):
    """Time the fp64 oracle on a sample of (sequence, head) pairs of the
    workload, growing the sample until about `budget_s` seconds."""
    import numpy as np

    import oracle
    inp = W.build_config(name, seed=seed, device="cpu")

    def to_f64(t):
        fmt = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float8_e4m3fn: "e4m3",
               torch.float8_e5m2: "e5m2"}[t.dtype]
        bits = (t.view(torch.int16).numpy().view(np.uint16) if t.element_size() == 2
                else t.view(torch.uint8).numpy())
        return oracle.decode(bits, fmt)

    q, k, v = to_f64(inp.q), to_f64(inp.k), to_f64(inp.v)
    sink = None if inp.sink is None else inp.sink.numpy()
    D = inp.head_dim
    pairs_done = 0
    heads = [(b, h) for h in range(inp.num_heads_q) for b in range(inp.batch)]
    rng = np.random.default_rng(seed)
    rng.shuffle(heads)
    t0 = time.perf_counter()
    n = 0
    for b, h in heads:
        rows = [(b, i, h) for i in range(inp.seqlens_q[b])]
        if inp.varlen:
            oracle.attention_varlen(q, k, v, inp.cu_seqlens_q.numpy(), inp.cu_seqlens_k.numpy(),
                                    inp.scale, inp.causal, inp.window, sink, rows=rows)
        else:
            oracle.attention_padded(q, k, v, inp.scale, inp.causal, inp.window, sink, rows=rows)
        pairs_done += _visible_pairs(inp.seqlens_q[b], inp.seqlens_k[b], inp.causal,
                                     inp.window[0], inp.window[1])
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    flops = 2.0 * (D + D) * pairs_done
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    try:
        host_cores = len(os.sched_getaffinity(0))
    except AttributeError:
        host_cores = os.cpu_count()
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
            "host_cores": host_cores, "host_cpu_count": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} of {len(heads)} (sequence, head) pairs, all query rows, "
                      f"{dt:.1f} s fp64 numpy"}


# ---------------------------------------------------------------------------
# timing
# ---------------------------------------------------------------------------

def load_for(fn, stream, seconds: float):
    """Untimed repetitions of a step for about `seconds`."""
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t0 < seconds:
            for _ in range(8):
                fn(stream)
            stream.synchronize()


def reduce_max_over_ranks(values_ms, world: int, device) -> list:
    """Max of each timing over all ranks (every rank gets the result)."""
    if world <= 1:
        return [float(v) for v in values_ms]
    t = torch.tensor([float(v) for v in values_ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(work_per_step: float, steps: int, world: int, total_ms: float) -> float:
    """Work done by all ranks (weak scaling: each rank runs `steps` steps of
    its own batch) divided by the slowest rank's time."""
    return work_per_step * steps * world / (total_ms / 1e3)


def time_steps(fn, steps: int, warmup: int, stream, flush):
    for _ in range(warmup):
        fn(stream)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with torch.cuda.stream(stream):
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            fn(stream)
            b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def run_ours(args, rank, world, device):
    stream = torch.cuda.Stream(device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    peaks, peak_kind = load_peaks()
    traffic = load_traffic()
    if args.all:
        names = list(args.only or WORKLOADS)
    elif args.headline_only or args.workload != HEADLINE:
        names = [args.workload]
    else:
        names = [args.workload] + DEFAULT_EXTRA
    if args.workload not in names:
        names.insert(0, args.workload)
    results = {}
    for name in names:
        wl = WORKLOADS[name](name, args.seed + rank, device)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        with ClockSampler(torch.cuda.current_device()) as clk:
            # Sampling runs through the warm-up and the timed steps. The timed
            # region is milliseconds long, shorter than the sampling period, so
            # the same step keeps the GPU busy for a short window right after
            # it, and those samples describe the clocks under this load. The
            # window comes after the timed steps, not before: a second of load
            # ahead of them would put the GPU at its power cap for the timed
            # steps, and the roofline divides by the burst peak.
            if args.clock_window > 0:
                clk.wait_first(3.0)
            times = time_steps(wl["step"], args.steps, args.warmup, stream, flush)
            if args.clock_window > 0:
                load_for(wl["step"], stream, args.clock_window)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        err = B.device_error(stream)
        if err:
            raise RuntimeError(f"{name}: device error word {err:#x}")
        e2e_times = time_steps(wl["e2e_step"], max(2, args.steps // 2), 2, stream, flush)
        tot, e2e_tot = reduce_max_over_ranks([sum(times), sum(e2e_times)], world, device)
        value = whole_job_rate(wl["work"], args.steps, world, tot)
        e2e_value = whole_job_rate(wl["work"], len(e2e_times), world, e2e_tot)
        per_launch = tot / args.steps / 1e3  # s, one kernel sequence
        achieved = wl["work"] / per_launch
        if wl["bound"] == "tensor":
            peak = peaks["bf16_tflops"] * (2.0 if wl["dtype"] in ("e4m3", "e5m2") else 1.0)
            runit = "TFLOP/s"
        else:
            peak = peaks["hbm_gbs"]
            runit = "GB/s"
        tr = traffic.get(wl["kernel"])
        tr_val = (tr["bytes_per_launch"]
                  if tr and tr.get("source_hash") == source_hash(wl["kernel"]) else None)
        results[name] = {
            "value": value, "unit": wl["unit"], "ms_per_step": tot / args.steps,
            "roofline": {"bound": wl["bound"], "achieved": achieved, "peak": peak, "unit": runit,
                         "frac": achieved / peak, "traffic": tr_val,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)"
                         if peak_kind == "measured" else "fallback"},
            "e2e": {"value": e2e_value, "unit": wl["unit"], "h2d_bytes_per_step": wl["h2d"],
                    "d2h_bytes_per_step": wl["d2h"]},
            "clocks": clk.summary(), "config": wl["cfg"], "dtype": wl["dtype"],
            "gpu_launches": wl["launches_per_step"] * args.steps,
            "work_per_step": wl["work"], "per_unit": wl["per_unit"],
        }
        if "gbytes" in wl:
            results[name]["gbytes_per_s"] = wl["gbytes"] / per_launch
            results[name]["hbm_frac"] = wl["gbytes"] / per_launch / peaks["hbm_gbs"]
        del wl
        torch.cuda.empty_cache()
    return results


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=list(WORKLOADS))
    ap.add_argument("--only", nargs="*", default=None, help="with --all: a subset of workloads")
    ap.add_argument("--all", action="store_true", help="also run every other workload")
    ap.add_argument("--headline-only", action="store_true",
                    help="time the headline workload alone (no decode / MLA / FP8 rows)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-window", type=float, default=0.5,
                    help="seconds of untimed load around the timed region while clocks are "
                         "sampled (0: none, e.g. under a profiler)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # The reference arm is the oracle, timed on the host cores of rank 0.
        if rank != 0:
            return
        base = cpu_baseline(args.workload, args.seed, args.cpu_budget)
        line = {"metric": METRIC, "value": base["value"], "unit": base["unit"], "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": args.workload, "l2": "n/a (host)"},
                "cpu_baseline": base,
                "e2e": {"value": base["value"], "unit": base["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    B.lib()
    res = run_ours(args, rank, world, device)
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(args.workload, args.seed, args.cpu_budget)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    h = res[args.workload]
    line = {
        "metric": METRIC, "value": h["value"], "unit": h["unit"], "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": h["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": h["dtype"],
        "data": "synthetic (seeded N(0,1) inputs of the workload's shapes)",
        "config": dict(h["config"], l2="flushed (512 MiB write) between timed steps",
                       parallelism=f"replicas x{world} (weak scaling, no collective)"),
        "roofline": h["roofline"], "e2e": h["e2e"], "clocks": h["clocks"],
        "gpu_launches": h["gpu_launches"], "cpu_baseline": base,
        "workloads": {k: {kk: vv for kk, vv in v.items() if kk != "config"} | {"config": v["config"]}
                      for k, v in res.items() if k != args.workload},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
