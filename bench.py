#!/usr/bin/env python
"""Benchmark of one paged-KV decode step on B200.

A step is one pass of the whole hot path over one batch: copy-on-write block
copies (when the workload has any), the slot-mapped write of one new token per
sequence, and paged decode attention (plan + attention + split-K reduce
kernels).  The default workload is the Llama-2-13B-shaped continuous batch
(B 128, 40 MHA heads, d 128, block size 16, fragmented pool).

Prints one JSON line.  `value` is algorithmic HBM GB/s of the whole step over
all ranks (bytes that must move: unique K/V rows read, q, out, tables and
lengths, the written rows and the copied blocks), measured with CUDA events on
inputs already resident in HBM; `e2e` is the same metric with the per-step
inputs copied from pinned host memory and the output copied back inside the
timed region.  `roofline` reports the decode call alone against the measured
HBM copy bandwidth.  `--impl reference` times the fp64 CPU oracle on the host
cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
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

import workloads  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.txt")
DECODE_SOURCES = ["paged_kv_cache_420_b200/csrc/decode.cuh", "paged_kv_cache_420_b200/csrc/ptx.cuh"]


# --------------------------------------------------------------------------
# algorithmic bytes
# --------------------------------------------------------------------------

def decode_bytes(w, kv_elem: int = 2) -> int:
    """Bytes paged decode attention must move: every distinct (block, kv head,
    offset) K and V row of valid tokens once (kv_elem bytes per element: 2 for
    bf16, 1 for an FP8 pool), q and out, the table entries read and the
    context lengths."""
    bs = w.block_size
    NB = w.num_blocks
    used = np.zeros((NB, bs), dtype=bool)
    for s in range(w.num_seqs):
        n = int(w.context_lens[s])
        nb = (n + bs - 1) // bs
        full = nb - 1
        if full > 0:
            used[w.block_tables[s, :full]] = True
        if nb > 0:
            used[w.block_tables[s, nb - 1], : n - full * bs] = True
    token_rows = int(used.sum())
    kv = token_rows * w.num_kv_heads * w.head_dim * kv_elem * 2
    qo = 2 * w.num_seqs * w.num_q_heads * w.head_dim * 2
    tables = 4 * int(sum((int(n) + bs - 1) // bs for n in w.context_lens))
    return kv + qo + tables + 4 * w.num_seqs


def logical_decode_bytes(w) -> int:
    """Same, but shared blocks counted once per sequence that reads them."""
    kv = int(w.context_lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 2 * 2
    qo = 2 * w.num_seqs * w.num_q_heads * w.head_dim * 2
    return kv + qo + 4 * int(sum((int(n) + w.block_size - 1) // w.block_size for n in w.context_lens)) + 4 * w.num_seqs


def write_bytes(w) -> int:
    return 2 * 2 * w.num_seqs * w.num_kv_heads * w.head_dim * 2 + 8 * w.num_seqs


def copy_bytes(w) -> int:
    blk = w.num_kv_heads * w.block_size * w.head_dim * 2
    return 2 * 2 * len(w.copy_pairs) * blk


def step_bytes(w) -> int:
    return decode_bytes(w) + write_bytes(w) + copy_bytes(w)


# --------------------------------------------------------------------------
# environment helpers
# --------------------------------------------------------------------------

def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, bs: int):
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken on the current decode sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 4 and not line.startswith("#"):
                    if parts[0] == decode_source_hash() and parts[1] == workload and parts[2] == f"bs{bs}":
                        return int(float(parts[3]))
    except FileNotFoundError:
        pass
    return None


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.text = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.text, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.text, _ = self.proc.communicate()

    def summary(self):
        if not getattr(self, "text", ""):
            return None
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.text.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# --------------------------------------------------------------------------
# the timed arms
# --------------------------------------------------------------------------

def combine_ranks(dist, ms_total: float, bytes_step: int, seqs: int, device):
    """Slowest rank's time, and all ranks' bytes and sequences per step."""
    if dist is None:
        return float(ms_total), float(bytes_step), float(seqs)
    stats = torch.tensor([ms_total, float(bytes_step), float(seqs)], dtype=torch.float64, device=device)
    mx = stats.clone()
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    sm = stats.clone()
    dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return float(mx[0]), float(sm[1]), float(sm[2])


def whole_job_gbs(bytes_all_ranks: float, steps: int, ms_max: float) -> float:
    """GB/s of the whole job: every rank's bytes over the slowest rank's time."""
    return bytes_all_ranks * steps / (ms_max / 1e3) / 1e9


def timed_passes(dev, stream, step, steps: int, dist):
    """Two timed passes of `steps` steps, clocks sampled over both.

    The first records only its two end events and gives the step time; the
    second calls step(i), which records an event pair around the kernel the
    roofline is about.  An event between two launches costs about 2 us of
    idle device time, so those events stay out of the first pass.
    Returns (ms of the first pass, ClockSampler).
    """
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        for i in range(steps):
            step(i)
        torch.cuda.synchronize()
        # keep sampling a little if the timed region was shorter than one sample
        if t0.elapsed_time(t1) < 450:
            time.sleep(0.45)
    return t0.elapsed_time(t1), clocks


def make_workload(args, rank: int, device):
    bs = args.block_size
    w = workloads.make(args.workload, seed=args.seed + rank, values_device=device, block_size=bs)
    if args.max_seqs and args.max_seqs < w.num_seqs:
        w = workloads.subset(w, args.max_seqs)
    return w


def partition_tokens(args, w) -> int:
    return w.partition_tokens if args.partition_tokens < 0 else args.partition_tokens


def library_partition_tokens(pt: int, max_context_len: int) -> int:
    """The partition size the library uses for `pt` (0 = its own choice)."""
    return pt if pt > 0 else (2048 if max_context_len > 16384 else 512)


def launches_per_step(w, pt: int) -> int:
    maxp = max(1, math.ceil(w.max_context_len / library_partition_tokens(pt, w.max_context_len)))
    n = 1 + 1 + 1 + (1 if maxp > 1 else 0)  # write, plan, attention, reduce
    if len(w.copy_pairs):
        n += math.ceil(len(w.copy_pairs) / 1024)
    return n


def run_cuda(args, rank, world, dist):
    import paged_kv_cache_420_b200 as pkv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = make_workload(args, rank, dev)
    pt = partition_tokens(args, w)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(w.q)
    ws = torch.empty(pkv.decode_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                                w.max_context_len, pt), dtype=torch.uint8, device=dev)
    kc, vc = w.k_cache, w.v_cache
    stream = torch.cuda.current_stream()
    ev_d = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def step(i=None):
        if len(w.copy_pairs):
            pkv.pkv_copy_blocks(w.copy_pairs, kc, vc, stream=stream)
        pkv.pkv_write(w.k_new, w.v_new, slots, kc, vc, stream=stream)
        if i is not None:
            ev_d[i][0].record(stream)
        pkv.paged_attn_decode(w.q, kc, vc, tables, ctx, w.scale, w.num_kv_heads, out, w.max_context_len, pt,
                              workspace=ws, stream=stream)
        if i is not None:
            ev_d[i][1].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    err = pkv.get_device_error()
    if err:
        raise RuntimeError(f"device error word {err:#x} during warm-up")

    ms_total, clocks = timed_passes(dev, stream, step, args.steps, dist)
    decode_ms = sum(a.elapsed_time(b) for a, b in ev_d) / args.steps
    if pkv.get_device_error():
        raise RuntimeError("device error word set during the timed region")

    bytes_step = step_bytes(w)
    dec_bytes = decode_bytes(w)
    ms_max, bytes_all, seqs_all = combine_ranks(dist, ms_total, bytes_step, w.num_seqs, dev)
    sec = ms_max / 1e3
    value = whole_job_gbs(bytes_all, args.steps, ms_max)

    # ---- end to end: per-step inputs from pinned host memory, output back
    e2e = None
    if not args.no_e2e:
        # Per step: the step's inputs are copied from pinned host memory and the
        # output back, inside the timed region.  Copies run on a second stream,
        # double-buffered, so step i+1's inputs and step i-1's output move
        # while step i computes (the kernels themselves stay in stream order).
        host = {k: v.cpu().pin_memory() for k, v in dict(q=w.q, k_new=w.k_new, v_new=w.v_new, slots=slots,
                                                           tables=tables, ctx=ctx).items()}
        dbuf = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
        dout = [torch.empty_like(out) for _ in range(2)]
        out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = out_h[0].numel() * out_h[0].element_size()
        k_e2e = max(3, args.steps)  # as long as the device-resident pass: same power state
        copy = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]

        def upload(i):
            b = i % 2
            if i >= 2:  # buffer b was read by step i-2
                copy.wait_event(ev_done[b])
            with torch.cuda.stream(copy):
                for k in host:
                    dbuf[b][k].copy_(host[k], non_blocking=True)
                ev_in[b].record(copy)

        def e2e_run(n):
            upload(0)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    upload(i + 1)  # the next step's inputs move while this step computes
                stream.wait_event(ev_in[b])
                if len(w.copy_pairs):
                    pkv.pkv_copy_blocks(w.copy_pairs, kc, vc, stream=stream)
                pkv.pkv_write(dbuf[b]["k_new"], dbuf[b]["v_new"], dbuf[b]["slots"], kc, vc, stream=stream)
                pkv.paged_attn_decode(dbuf[b]["q"], kc, vc, dbuf[b]["tables"], dbuf[b]["ctx"], w.scale,
                                      w.num_kv_heads, dout[b], w.max_context_len, pt, workspace=ws, stream=stream)
                ev_done[b].record(stream)
                copy.wait_event(ev_done[b])
                with torch.cuda.stream(copy):
                    out_h[b].copy_(dout[b], non_blocking=True)

        e2e_run(4)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as e2e_clocks:
            a.record(copy)
            stream.wait_stream(copy)
            e2e_run(k_e2e)
            copy.wait_stream(stream)
            b_.record(copy)
            torch.cuda.synchronize()
        if not torch.equal(out_h[(k_e2e - 1) % 2].to(dev), out):
            raise RuntimeError("end-to-end output differs from the device-resident run")
        e_ms = torch.tensor([a.elapsed_time(b_)], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
        e2e = {"value": round(bytes_all * k_e2e / (float(e_ms[0]) / 1e3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": k_e2e,
               "overlap": "copies on a second stream, double-buffered", "clocks": e2e_clocks.summary()}

    peak, peak_kind = measured_hbm_peak()
    achieved = dec_bytes / (decode_ms / 1e3) / 1e9
    line = {
        "metric": "paged decode attn HBM GB/s (% of B200 peak) & tokens·layers/s at 13B shape",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"{w.name}: {w.description}",
            "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size, "kv_tokens": int(w.context_lens.sum()),
            "partition_tokens": library_partition_tokens(pt, w.max_context_len), "copy_pairs": int(len(w.copy_pairs)),
            "seed": args.seed, "bytes_per_step": int(bytes_step),
            "l2": "no flush: every step reads >1 GB of K/V (L2 is 126 MB)",
            "parallelism": f"replicas x{world}, one independent batch per GPU",
        },
        "tokens_layers_per_s": round(seqs_all * args.steps / sec, 1),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "roofline": {
            "kernel": "paged_attn_decode (plan + attention + reduce kernels)",
            "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind,
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "algorithmic_bytes": int(dec_bytes), "logical_bytes": int(logical_decode_bytes(w)),
            "decode_us": round(decode_ms * 1e3, 2),
            "traffic": recorded_traffic(w.name, w.block_size),
        },
        "e2e": e2e,
        "gpu_launches": launches_per_step(w, pt) * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget,
                                            single_thread_s=3.0 if w.name in SINGLE_THREAD_WORKLOADS else 0.0)
    if world == 1 and not args.no_shapes and w.name == "llama2-13b" and not args.max_seqs:
        del w, kc, vc, out, ws
        torch.cuda.empty_cache()
        line["shapes"] = other_shapes(dev, stream)
    return line


# --------------------------------------------------------------------------
# decode-alone timings of the other shapes, reported beside the headline step
# --------------------------------------------------------------------------

L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2
COPY_SLEEP_CYCLES = 400_000  # about 0.2 ms of device time


def time_calls(fn, stream, n: int, warm: int = 5, between=None):
    """Median and mean CUDA-event time (us) of `fn` over n calls on `stream`,
    after `warm` untimed calls.  `between` (untimed, outside the events) runs
    before every call, e.g. an L2 flush."""
    for _ in range(warm):
        if between is not None:
            between()
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in ev:
        if between is not None:
            between()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    t = [1e3 * a.elapsed_time(b) for a, b in ev]
    return statistics.median(t), statistics.fmean(t)


def _timed_with_clocks(dev, fn, stream, n, warm=5, between=None):
    with ClockSampler(dev.index) as clocks:
        med, mean = time_calls(fn, stream, n, warm, between)
        time.sleep(0.45)  # at least two clock samples
    return med, mean, clocks.summary()


def decode_shape(pkv, dev, stream, name, bs, pt, peak, n=50, fp8=False, flush=None):
    """Decode attention alone (plan + attention + reduce) on one of the decode
    workloads, after its copy-on-write copies and write."""
    w = workloads.make(name, seed=0, values_device=dev, block_size=bs)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(w.q)
    ws = torch.empty(pkv.decode_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                                w.max_context_len, pt), dtype=torch.uint8, device=dev)
    if fp8:
        kc, vc, ks, vs = workloads.fp8_pools(w)
        del w.k_cache, w.v_cache
        if len(w.copy_pairs):
            pkv.pkv_copy_blocks(w.copy_pairs, kc, vc, stream=stream)
        pkv.pkv_write_fp8(w.k_new, w.v_new, slots, ks, vs, kc, vc, stream=stream)

        def call():
            pkv.paged_attn_decode_fp8(w.q, kc, vc, ks, vs, tables, ctx, w.scale, w.num_kv_heads, out,
                                      w.max_context_len, pt, workspace=ws, stream=stream)
    else:
        kc, vc = w.k_cache, w.v_cache
        if len(w.copy_pairs):
            pkv.pkv_copy_blocks(w.copy_pairs, kc, vc, stream=stream)
        pkv.pkv_write(w.k_new, w.v_new, slots, kc, vc, stream=stream)

        def call():
            pkv.paged_attn_decode(w.q, kc, vc, tables, ctx, w.scale, w.num_kv_heads, out, w.max_context_len, pt,
                                  workspace=ws, stream=stream)
    med, mean, clk = _timed_with_clocks(dev, call, stream, n, between=flush)
    if pkv.get_device_error():
        raise RuntimeError(f"device error word set on {name}")
    nbytes = decode_bytes(w, kv_elem=1 if fp8 else 2)
    gbs = nbytes / (med * 1e-6) / 1e9
    rec = {"workload": f"{w.name}: {w.description}", "kv": "e4m3" if fp8 else "bf16", "block_size": w.block_size,
           "partition_tokens": library_partition_tokens(pt, w.max_context_len), "decode_us": round(med, 2),
           "decode_us_mean": round(mean, 2), "algorithmic_bytes": int(nbytes), "achieved_gbs": round(gbs, 1),
           "frac": round(gbs / peak, 4), "calls": n, "clocks": clk}
    if w.name == "llama3-8b-gqa-prefix":
        rec["logical_bytes"] = int(logical_decode_bytes(w))
    del w, kc, vc, out, ws
    torch.cuda.empty_cache()
    return rec


def prefill_shape(pkv, dev, stream, name, tpeak, n=30):
    w = workloads.make_prefill(name, seed=0, values_device=dev)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    qs = torch.from_numpy(w.query_start).to(dev)
    out = torch.empty_like(w.q)
    ws = torch.empty(pkv.prefill_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.max_query_len),
                     dtype=torch.uint8, device=dev)
    pkv.pkv_write(w.k_new, w.v_new, slots, w.k_cache, w.v_cache, stream=stream)

    def call():
        pkv.paged_attn_prefill(w.q, w.k_cache, w.v_cache, tables, ctx, qs, w.scale, w.num_kv_heads, out,
                               w.max_query_len, w.max_context_len, workspace=ws, stream=stream)
    med, mean, clk = _timed_with_clocks(dev, call, stream, n)
    if pkv.get_device_error():
        raise RuntimeError(f"device error word set on {name}")
    flops = prefill_flops(w)
    tf = flops / (med * 1e-6) / 1e12
    rec = {"workload": f"{w.name}: {w.description}", "prefill_us": round(med, 2), "prefill_us_mean": round(mean, 2),
           "algorithmic_flops": flops, "achieved_tflops": round(tf, 1), "frac": round(tf / tpeak, 4), "calls": n,
           "clocks": clk}
    del w, out, ws
    torch.cuda.empty_cache()
    return rec


def copy_shape(pkv, dev, stream, peak, flush, pairs=256, n=50):
    """pkv_copy_blocks on `pairs` copy-on-write pairs of the Llama-3-8B block
    shape (8 kv heads x 16 tokens x 128, bf16: 32 KB of K and 32 KB of V per
    block), sources and destinations distinct, L2 flushed before each call."""
    rng = np.random.default_rng(7)
    nb = 4 * pairs
    kc = torch.randn(nb, 8, 16, 128, device=dev).to(torch.bfloat16)
    vc = torch.randn(nb, 8, 16, 128, device=dev).to(torch.bfloat16)
    ids = rng.permutation(nb)[:2 * pairs].astype(np.int32)
    cp = np.stack([ids[:pairs], ids[pairs:]], axis=1)
    # The call validates its pairs on the host (sorts and searches); for long
    # lists that takes longer than the flush, and the device would sit idle
    # inside the timed region.  A device sleep after the flush lets the host
    # enqueue the call first, so the events time the kernel alone.
    def between():
        flush()
        torch.cuda._sleep(COPY_SLEEP_CYCLES)

    med, mean, clk = _timed_with_clocks(dev, lambda: pkv.pkv_copy_blocks(cp, kc, vc, stream=stream), stream, n,
                                        between=between)
    blk = kc[0].numel() * 2
    nbytes = 2 * 2 * pairs * blk  # K and V, read and written
    gbs = nbytes / (med * 1e-6) / 1e9
    del kc, vc
    torch.cuda.empty_cache()
    return {"workload": f"{pairs} pairs of {2 * blk // 1024} KB blocks (K+V), 8 kv heads, bs16, d128",
            "copy_us": round(med, 2), "copy_us_mean": round(mean, 2), "algorithmic_bytes": nbytes,
            "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "calls": n,
            "l2": "256 MB read before each call", "timing": "a device sleep before each start event hides the host-side validation",
            "clocks": clk}


def other_shapes(dev, stream):
    """Decode alone at the GQA and long-context shapes (512-token partitions as
    specified), the 13B decode with and without an L2 flush between calls, the
    FP8 decode, the chunked prefill and block copies of 256 and 1024 pairs.  Each record
    carries its own clocks; none of them enters the headline value."""
    import paged_kv_cache_420_b200 as pkv

    peak, _ = measured_hbm_peak()
    tpeak, _ = measured_tensor_peak()
    scratch = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)

    def flush():
        # a read of twice the L2 size: L2 then holds clean lines of the scratch
        # (a write would leave dirty lines whose write-back the next call pays)
        scratch.sum()

    shapes = {}
    for key, name, bs, pt in (("llama3-8b-gqa-prefix", "llama3-8b-gqa-prefix", 16, 0),
                              ("llama2-70b-long bs16", "llama2-70b-long", 16, 512),
                              ("llama2-70b-long bs128", "llama2-70b-long", 128, 512),
                              ("llama2-7b", "llama2-7b", 16, 0)):
        shapes[key] = decode_shape(pkv, dev, stream, name, bs, pt, peak)
    shapes["llama2-13b l2-flushed"] = decode_shape(pkv, dev, stream, "llama2-13b", 16, 0, peak, flush=flush)
    shapes["llama2-13b l2-flushed"]["l2"] = "256 MB read before each call"
    shapes["llama2-13b unflushed"] = decode_shape(pkv, dev, stream, "llama2-13b", 16, 0, peak)
    shapes["llama2-13b-fp8"] = decode_shape(pkv, dev, stream, "llama2-13b", 16, 0, peak, fp8=True)
    shapes["llama3-8b-gqa-prefix-fp8"] = decode_shape(pkv, dev, stream, "llama3-8b-gqa-prefix", 16, 0, peak,
                                                      fp8=True)
    for name in workloads.PREFILL_WORKLOADS:
        shapes[name] = prefill_shape(pkv, dev, stream, name, tpeak)
    shapes["copy_blocks 256 pairs"] = copy_shape(pkv, dev, stream, peak, flush)
    shapes["copy_blocks 1024 pairs"] = copy_shape(pkv, dev, stream, peak, flush, pairs=1024)
    del scratch
    torch.cuda.empty_cache()
    return shapes


def prefill_flops(w) -> float:
    """QK^T and PV multiply-adds of causal chunked prefill: every (query row,
    query head) attends to pos + 1 keys, 2 flops per element of each."""
    keys = 0
    for s in range(w.num_seqs):
        ql = int(w.query_start[s + 1] - w.query_start[s])
        n = int(w.context_lens[s])
        keys += ql * (n - ql) + ql * (ql + 1) // 2
    return 4.0 * w.head_dim * w.num_q_heads * keys


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def run_prefill_cuda(args, rank, world, dist):
    """One step = slot-mapped write of every chunk token + chunked-prefill
    attention; metric TFLOP/s of the attention (causal flops)."""
    import paged_kv_cache_420_b200 as pkv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workloads.make_prefill(args.workload, seed=args.seed + rank, values_device=dev, block_size=args.block_size)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    qs = torch.from_numpy(w.query_start).to(dev)
    out = torch.empty_like(w.q)
    ws = torch.empty(pkv.prefill_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.max_query_len),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def step(i=None):
        pkv.pkv_write(w.k_new, w.v_new, slots, w.k_cache, w.v_cache, stream=stream)
        if i is not None:
            ev[i][0].record(stream)
        pkv.paged_attn_prefill(w.q, w.k_cache, w.v_cache, tables, ctx, qs, w.scale, w.num_kv_heads, out,
                               w.max_query_len, w.max_context_len, workspace=ws, stream=stream)
        if i is not None:
            ev[i][1].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    ms_run, clocks = timed_passes(dev, stream, step, args.steps, dist)
    if pkv.get_device_error():
        raise RuntimeError("device error word set during the timed region")
    flops = prefill_flops(w)
    ms_max, flops_all, tok_all = combine_ranks(dist, ms_run, int(flops), w.num_tokens, dev)
    attn_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    peak, kind = measured_tensor_peak()
    achieved = flops / (attn_ms / 1e3) / 1e12
    return {
        "metric": "paged chunked-prefill attention TFLOP/s",
        "value": round(flops_all * args.steps / (ms_max / 1e3) / 1e12, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.description}", "num_seqs": w.num_seqs,
                   "query_tokens": w.num_tokens, "kv_tokens": int(w.context_lens.sum()),
                   "block_size": w.block_size, "seed": args.seed},
        "tokens_per_s": round(tok_all * args.steps / (ms_max / 1e3), 1),
        "roofline": {"kernel": "paged_attn_prefill (plan + attention kernels)", "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": peak, "peak_kind": kind, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "algorithmic_flops": flops,
                     "prefill_us": round(attn_ms * 1e3, 2), "traffic": None},
        "e2e": None, "gpu_launches": 3 * args.steps, "clocks": clocks.summary(),
    }


SWAP_WORKLOADS = ("llama2-13b-swap",)
FP8_WORKLOADS = ("llama2-13b-fp8", "llama3-8b-gqa-prefix-fp8")


def run_fp8_cuda(args, rank, world, dist):
    """A decode step on an FP8 (e4m3) pool (the Llama-2-13B batch, or the
    Llama-3-8B shared-prefix batch): the quantizing write of each sequence's
    new token, then decode attention over the e4m3 codes with per-kv-head K/V
    scales, after the batch's copy-on-write copies (if any).  Metric:
    algorithmic HBM GB/s of the step (one byte per cached element) and
    tokens*layers/s, comparable with the bf16 step's."""
    import paged_kv_cache_420_b200 as pkv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    base = args.workload[:-len("-fp8")]
    w = workloads.make(base, seed=args.seed + rank, values_device=dev, block_size=args.block_size)
    if args.max_seqs and args.max_seqs < w.num_seqs:
        w = workloads.subset(w, args.max_seqs)
    k8, v8, ks, vs = workloads.fp8_pools(w)
    del w.k_cache, w.v_cache
    torch.cuda.empty_cache()
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(w.q)
    mctx = int(w.context_lens.max())
    ws = torch.empty(pkv.decode_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, mctx),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def step(i=None):
        if len(w.copy_pairs):
            pkv.pkv_copy_blocks(w.copy_pairs, k8, v8, stream=stream)
        pkv.pkv_write_fp8(w.k_new, w.v_new, slots, ks, vs, k8, v8, stream=stream)
        if i is not None:
            ev[i][0].record(stream)
        pkv.paged_attn_decode_fp8(w.q, k8, v8, ks, vs, tables, ctx, w.scale, w.num_kv_heads, out, mctx,
                                  workspace=ws, stream=stream)
        if i is not None:
            ev[i][1].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    ms_run, clocks = timed_passes(dev, stream, step, args.steps, dist)
    if pkv.get_device_error():
        raise RuntimeError("device error word set during the timed region")
    dec = decode_bytes(w, kv_elem=1)
    wr = w.num_seqs * w.num_kv_heads * w.head_dim * (2 * 2 + 2) + 8 * w.num_seqs  # bf16 in, e4m3 out
    wr += copy_bytes(w) // 2  # e4m3 blocks
    ms_max, bytes_all, seqs_all = combine_ranks(dist, ms_run, dec + wr, w.num_seqs, dev)
    dec_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    peak, kind = measured_hbm_peak()
    achieved = dec / (dec_ms / 1e3) / 1e9
    # copies (when the batch has pairs), write, plan, attention, and the
    # split-K reduce when some context spans more than one partition
    launches = (1 if len(w.copy_pairs) else 0) + 3 + (1 if mctx > library_partition_tokens(0, mctx) else 0)
    return {
        "metric": f"paged decode attn HBM GB/s on an FP8 (e4m3) pool & tokens*layers/s ({base})",
        "value": whole_job_gbs(bytes_all, args.steps, ms_max), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 KV, bf16 q/out",
        "data": "synthetic",
        "config": {"workload": f"{w.name} with an FP8 pool: {w.description}", "block_size": w.block_size,
                   "num_seqs": w.num_seqs, "seed": args.seed},
        "tokens_layers_per_s": round(seqs_all * args.steps / (ms_max / 1e3), 1),
        "roofline": {"kernel": "paged_attn_decode_fp8 (plan + attention kernels)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "algorithmic_bytes": dec,
                     "decode_us": round(dec_ms * 1e3, 2), "traffic": None},
        "e2e": None, "gpu_launches": args.steps * launches, "clocks": clocks.summary(),
    }
BM_WORKLOADS = ("llama2-13b-blockmgr",)


def run_blockmgr_cuda(args, rank, world, dist):
    """Device block manager on the Llama-2-13B batch (128 sequences, their
    context lengths): one step = append_slots for one new token per sequence
    (block allocation as sequences cross a block boundary, slot mapping, copy-
    on-write checks), timed per call; a 512-token chunk per sequence for 8
    sequences is timed as the prefill case.  Metric: microseconds per decode
    step; the floor is an empty kernel's launch-to-completion on the same
    stream.  The CPU baseline is the oracle's sequential append on the host."""
    import oracle
    import paged_kv_cache_420_b200 as pkv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workloads.make("llama2-13b", seed=args.seed + rank, values_device="cpu", block_size=args.block_size)
    B, bs = w.num_seqs, w.block_size
    steps = args.steps
    mbs = (int(w.context_lens.max()) + steps + 2 * bs) // bs + 1
    nb = B * mbs + 64
    stream = torch.cuda.current_stream()

    def fresh():
        bm = pkv.BlockManager(nb, device=dev)
        t = torch.full((B, mbs), -1, dtype=torch.int32, device=dev)
        c = torch.zeros(B, dtype=torch.int32, device=dev)
        fill = torch.from_numpy(w.context_lens.astype(np.int32)).to(dev)
        bm.append_slots(t, c, fill, bs, int(w.context_lens.sum()))
        return bm, t, c

    bm, tables, ctx = fresh()
    one = torch.ones(B, dtype=torch.int32, device=dev)
    out = (torch.empty(B, dtype=torch.int64, device=dev), torch.empty((B, 2), dtype=torch.int32, device=dev),
           torch.empty(1, dtype=torch.int32, device=dev))
    for _ in range(max(args.warmup, 3)):
        bm.append_slots(tables, ctx, one, bs, B, out=out)
    torch.cuda.synchronize()
    # the steps go into CUDA graphs of 64 calls: the device time, not the
    # Python enqueue rate, is what is measured
    per_graph = 64
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(per_graph):
            bm.append_slots(tables, ctx, one, bs, B, out=out)
    torch.cuda.synchronize()
    reps = max(1, steps // per_graph)
    steps = reps * per_graph
    mbs_needed = (int(ctx.max().item()) + steps + bs) // bs
    if mbs_needed > mbs:
        raise RuntimeError("block-table rows too short for the timed steps")
    if dist is not None:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        t0.record(stream)
        for _ in range(reps):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        if t0.elapsed_time(t1) < 450:
            time.sleep(0.45)
    if bm.error():
        raise RuntimeError(f"block manager error word {bm.error():#x}")
    ms_max, _, _ = combine_ranks(dist, t0.elapsed_time(t1), B, B, dev)
    per_call_us = 1e3 * t0.elapsed_time(t1) / steps
    del graph
    # prefill-sized step: 8 sequences, 512 new tokens each
    bm2, t2, c2 = fresh()
    chunk = torch.zeros(B, dtype=torch.int32, device=dev)
    chunk[:8] = 512
    pre = []
    pout = (torch.empty(8 * 512, dtype=torch.int64, device=dev), torch.empty((B, 2), dtype=torch.int32, device=dev),
            torch.empty(1, dtype=torch.int32, device=dev))
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        bm2, t2, c2 = fresh()
        torch.cuda.synchronize()
        a.record(stream)
        bm2.append_slots(t2, c2, chunk, bs, 8 * 512, out=pout)
        b.record(stream)
        torch.cuda.synchronize()
        pre.append(a.elapsed_time(b) * 1e3)
    # prefix cache: 128 prompts of 512 tokens sharing a 256-token system prompt
    rng = np.random.default_rng(args.seed)
    system = rng.integers(0, 32000, 256)
    prompts = [np.concatenate([system, rng.integers(0, 32000, 256)]).astype(np.int32) for _ in range(B)]
    toks = torch.from_numpy(np.concatenate(prompts)).to(dev)
    qs = torch.from_numpy(np.arange(B + 1, dtype=np.int32) * 512).to(dev)
    pmbs = 512 // bs + 1
    bm3 = pkv.BlockManager(B * pmbs + 64, device=dev)
    pc = pkv.PrefixCache(1 << 16, device=dev)
    t3 = torch.full((B, pmbs), -1, dtype=torch.int32, device=dev)
    c3 = torch.zeros(B, dtype=torch.int32, device=dev)
    bm3.append_slots(t3, c3, torch.full((B,), 512, dtype=torch.int32, device=dev), bs, B * 512)
    pc.insert(bm3, toks, qs, bs, t3)  # the first batch fills the cache
    lk, ins = [], []
    for _ in range(5):
        tl = torch.full((B, pmbs), -1, dtype=torch.int32, device=dev)
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        cached = pc.lookup(bm3, toks, qs, bs, tl)
        b.record(stream)
        pc.insert(bm3, toks, qs, bs, t3)
        c.record(stream)
        torch.cuda.synchronize()
        lk.append(a.elapsed_time(b) * 1e3)
        ins.append(b.elapsed_time(c) * 1e3)
        bm3.free(tl[tl >= 0].contiguous())  # drop the lookup's references again
    prefix_hit_tokens = int(cached.sum().item())
    # floor: an empty kernel, launch to completion
    nop = torch.empty(1, device=dev)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        for _ in range(per_graph):
            nop.zero_()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(10):
        g2.replay()
    b.record(stream)
    torch.cuda.synchronize()
    floor_us = 1e3 * a.elapsed_time(b) / (10 * per_graph)
    del g2
    # CPU baseline: the oracle's sequential append for the same decode step
    st = oracle.bm_init(nb)
    ot = np.full((B, mbs), -1, np.int32)
    st, ot, oc, _, _, _ = oracle.bm_append_slots(st, ot, np.zeros(B, np.int32), w.context_lens.astype(np.int32), bs)
    ones = np.ones(B, np.int32)
    t = time.perf_counter()
    n_cpu = 0
    while time.perf_counter() - t < 2.0:
        st, ot, oc, _, _, _ = oracle.bm_append_slots(st, ot, oc, ones, bs)
        n_cpu += 1
        if int(oc.max()) + 1 >= mbs * bs:
            break
    cpu_us = (time.perf_counter() - t) / max(n_cpu, 1) * 1e6
    return {
        "metric": "device block-manager append_slots microseconds per decode step",
        "value": round(1e3 * ms_max / steps, 3), "unit": "us", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / steps, 5), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "int32", "data": "synthetic",
        "config": {"workload": f"llama2-13b batch: {B} sequences, bs {bs}, one new token each per step; "
                               f"prefill case 8 x 512 tokens", "block_size": bs, "seed": args.seed},
        "roofline": {"kernel": "bm_append_slots_kernel", "bound": "latency", "achieved": round(per_call_us, 2),
                     "peak": round(floor_us, 2),
                     "peak_kind": "measured: one-thread kernel per graph node, back to back (launch floor)",
                     "unit": "us", "frac": round(floor_us / per_call_us, 4),
                     "prefill_8x512_us": round(float(np.median(pre)), 2),
                     "prefix_lookup_128x512_us": round(float(np.median(lk)), 2),
                     "prefix_insert_128x512_us": round(float(np.median(ins)), 2),
                     "prefix_hit_tokens": prefix_hit_tokens, "traffic": None},
        "cpu_baseline": {"value": round(cpu_us, 2), "unit": "us", "cores": 1, "kind": "oracle",
                         "sample": f"{n_cpu} sequential append steps of the same batch"},
        "e2e": None, "gpu_launches": steps, "clocks": clocks.summary(),
    }


def run_swap_cuda(args, rank, world, dist):
    """One step = swap-out of the LRU victim blocks of the Llama-2-13B pool to
    pinned host memory, then swap-in of the same blocks (a preemption cycle,
    about 256 MB each way).  Metric: GB/s moved over the host link; the
    roofline peak is a plain pinned DMA copy of the same bytes (both ways),
    measured in the same run."""
    import paged_kv_cache_420_b200 as pkv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = workloads.make("llama2-13b", seed=args.seed + rank, values_device=dev, block_size=args.block_size)
    nb = w.k_cache.shape[0]
    rng = np.random.default_rng(args.seed + rank)
    # blocks of a sequence share its last scheduling time; unowned blocks are free
    owner_time = rng.permutation(w.num_seqs)
    last_use = np.zeros(nb, dtype=np.int64)
    evictable = np.zeros(nb, dtype=np.uint8)
    for s in range(w.num_seqs):
        nblk = (int(w.context_lens[s]) + w.block_size - 1) // w.block_size
        blk = w.block_tables[s, :nblk]
        last_use[blk] = owner_time[s]
        evictable[blk] = 1
    block_bytes = w.k_cache[0].numel() * 2
    k = int(min(evictable.sum(), max(1, round((256 << 20) / (2 * block_bytes)))))
    victims = pkv.lru_victims(last_use, evictable, k)
    n = len(victims)
    hk = torch.empty((n,) + tuple(w.k_cache.shape[1:]), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]

    def step(i=None):
        if i is not None:
            ev[i][0].record(stream)
        pkv.pkv_swap_out(w.k_cache, w.v_cache, victims, hk, hv, stream=stream)
        if i is not None:
            ev[i][1].record(stream)
        pkv.pkv_swap_in(hk, hv, victims, w.k_cache, w.v_cache, stream=stream)
        if i is not None:
            ev[i][2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    # the link: DMA copies of the same bytes, device -> pinned host and back
    dk = torch.empty((n,) + tuple(w.k_cache.shape[1:]), dtype=torch.bfloat16, device=dev)
    dv = torch.empty_like(dk)
    d2h_ms, h2d_ms = [], []
    for _ in range(5):
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        hk.copy_(dk, non_blocking=True)
        hv.copy_(dv, non_blocking=True)
        b.record(stream)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        c.record(stream)
        torch.cuda.synchronize()
        d2h_ms.append(a.elapsed_time(b))
        h2d_ms.append(b.elapsed_time(c))
    del dk, dv
    ms_run, clocks = timed_passes(dev, stream, step, args.steps, dist)
    bytes_step = 2 * n * block_bytes * 2  # K and V, out and in
    ms_max, bytes_all, _ = combine_ranks(dist, ms_run, bytes_step, n, dev)
    out_ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
    in_ms = float(np.median([e[1].elapsed_time(e[2]) for e in ev]))
    one_way = 2 * n * block_bytes
    dma_ms = float(np.median(d2h_ms)) + float(np.median(h2d_ms))
    achieved = bytes_step / ((out_ms + in_ms) / 1e3) / 1e9
    peak = bytes_step / (dma_ms / 1e3) / 1e9
    return {
        "metric": "block swap GB/s (out to pinned host memory and back in)",
        "value": round(bytes_all * args.steps / (ms_max / 1e3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"llama2-13b pool, {n} LRU victim blocks of {block_bytes * 2} B (K+V), "
                               f"{one_way / 1e6:.1f} MB each way", "block_size": w.block_size, "seed": args.seed},
        "roofline": {"kernel": "swap_blocks_kernel (out, in)", "bound": "host link",
                     "achieved": round(achieved, 2), "peak": round(peak, 2),
                     "peak_kind": "measured: pinned cudaMemcpyAsync of the same bytes, D2H then H2D",
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "swap_out_gbs": round(one_way / (out_ms / 1e3) / 1e9, 2),
                     "swap_in_gbs": round(one_way / (in_ms / 1e3) / 1e9, 2),
                     "dma_d2h_gbs": round(one_way / (float(np.median(d2h_ms)) / 1e3) / 1e9, 2),
                     "dma_h2d_gbs": round(one_way / (float(np.median(h2d_ms)) / 1e3) / 1e9, 2),
                     "traffic": None},
        "e2e": None, "gpu_launches": 2 * args.steps, "clocks": clocks.summary(),
    }


# workloads whose CPU baseline also reports a single-thread figure
SINGLE_THREAD_WORKLOADS = ("tiny", "llama2-7b")


def cpu_baseline(w, budget_s: float, label="oracle", pools=None, single_thread_s: float = 0.0):
    """Times the fp64 CPU oracle's paged attention on the first sequences of
    the workload until about `budget_s` seconds of CPU work are spent.  The
    step's copy-on-write copies and write are applied to the pools once,
    untimed (they are under 1% of the step's bytes).  With single_thread_s > 0
    the same is timed on one thread for about that long and reported as
    `single_thread`."""
    import oracle

    if pools is None:
        pools = oracle_pools(w)
    line = _time_oracle(w, budget_s, label, pools)
    if single_thread_s > 0:
        prev = oracle.set_num_threads(1)
        try:
            one = _time_oracle(w, single_thread_s, label, pools)
        finally:
            oracle.set_num_threads(prev)
        line["single_thread"] = {"value": one["value"], "unit": one["unit"], "cores": 1, "sample": one["sample"],
                                 "tokens_layers_per_s": one["tokens_layers_per_s"]}
    return line


def _time_oracle(w, budget_s: float, label, pools):
    import oracle

    kc, vc = pools
    done, elapsed, nbytes = 0, 0.0, 0
    chunk = 1
    while elapsed < budget_s:
        start = done % w.num_seqs
        idx = np.arange(start, min(w.num_seqs, start + chunk))
        sub = _subset(w, idx)
        t = time.perf_counter()
        oracle.paged_attention(sub.q, kc, vc, sub.block_tables, sub.context_lens, sub.scale)
        elapsed += time.perf_counter() - t
        nbytes += decode_bytes(sub)
        done += len(idx)
        chunk = min(2 * chunk, 64)
    passes = done / w.num_seqs
    return {"value": round(nbytes / elapsed / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": label,
            "sample": f"paged attention of {done} sequences ({passes:.2f} passes over the {w.num_seqs}-sequence "
                      f"batch, all heads), {elapsed:.1f} s of fp64 C/OpenMP work",
            "tokens_layers_per_s": round(done / elapsed, 2)}


def oracle_pools(w):
    """Pools after the step's copy-on-write copies and write, by the oracle."""
    import oracle

    kc, vc = oracle.bits(w.k_cache), oracle.bits(w.v_cache)
    if len(w.copy_pairs):
        kc, vc = oracle.copy_blocks(kc, vc, w.copy_pairs)
    return oracle.kv_write(kc, vc, w.k_new, w.v_new, w.slot_mapping)


def _subset(w, idx):
    import copy as _copy
    sub = _copy.copy(w)
    ti = torch.from_numpy(np.asarray(idx, dtype=np.int64)).to(w.q.device)
    sub.q, sub.k_new, sub.v_new = w.q[ti], w.k_new[ti], w.v_new[ti]
    sub.block_tables = w.block_tables[idx]
    sub.context_lens = w.context_lens[idx]
    sub.slot_mapping = w.slot_mapping[idx]
    sub.num_seqs = len(idx)
    if len(w.copy_pairs):
        dsts = set(int(b) for b in np.unique(sub.block_tables))
        sub.copy_pairs = np.array([p for p in w.copy_pairs if int(p[1]) in dsts], np.int32).reshape(-1, 2)
    return sub


def run_prefill_reference(args, world):
    """The CPU oracle's chunked prefill on the host cores: each step is a
    bounded sample of query rows (whole sequences' chunks, cycling)."""
    import oracle

    w = workloads.make_prefill(args.workload, seed=args.seed, values_device="cpu", block_size=args.block_size)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    budget = max(0.05, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    qb = oracle.bits(w.q)
    vals, t_all, rows_done, flops_done, spent, seq = [], 0.0, 0, 0.0, 0.0, 0
    for i in range(args.warmup + args.steps):
        spent_step, fl = 0.0, 0.0
        while spent_step < budget:
            s = seq % w.num_seqs
            a, b = int(w.query_start[s]), int(w.query_start[s + 1])
            rows = np.arange(a, min(b, a + 16))  # 16 query rows of the chunk
            pos = w.context_lens[s] - (b - rows)
            ctx = (pos + 1).astype(np.int32)
            t = time.perf_counter()
            oracle.paged_prefill(qb[rows], kc, vc, w.block_tables[[s] * len(rows)], ctx,
                                 np.arange(len(rows) + 1, dtype=np.int32), w.scale)
            spent_step += time.perf_counter() - t
            fl += 4.0 * w.head_dim * w.num_q_heads * float(ctx.sum())
            seq += 1
            if i >= args.warmup:
                rows_done += len(rows)
        if i >= args.warmup:
            vals.append(fl / spent_step / 1e12)
            t_all += spent_step
    value = statistics.median(vals)
    return {
        "impl": "reference", "metric": "paged chunked-prefill attention TFLOP/s", "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_all / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.description}", "seed": args.seed},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{rows_done} query rows (16 per sequence, cycling), all heads"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_swap_reference(args, world):
    """The oracle's swap-out and swap-in (plain C loops over host arrays) on a
    sample with the Llama-2-13B block shape: 128 of 512 blocks out and back in."""
    import oracle

    rng = np.random.default_rng(args.seed)
    shape = (512, 40, args.block_size or 16, 128)
    kc = rng.integers(0, 1 << 16, size=shape, dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=shape, dtype=np.uint16)
    ids = rng.permutation(shape[0])[:128].astype(np.int32)
    block_bytes = int(np.prod(shape[1:])) * 2
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        hk, hv = oracle.swap_out(kc, vc, ids)
        kc, vc = oracle.swap_in(kc, vc, hk, hv, ids)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    bytes_step = 2 * len(ids) * block_bytes * 2
    value = round(bytes_step / statistics.median(times) / 1e9, 3)
    sample = f"{len(ids)} of {shape[0]} blocks of shape {shape[1:]}, out and back in, per step"
    return {
        "impl": "reference", "metric": "block swap GB/s (out to pinned host memory and back in)",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16", "data": "synthetic",
        "config": {"workload": "llama2-13b block shape swap sample", "block_size": shape[2], "seed": args.seed},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_fp8_reference(args, world):
    """The oracle's FP8 attention (fp64) on the first sequences of the 13B
    batch with an FP8 pool, in the GPU line's unit (algorithmic GB/s)."""
    import oracle

    w = workloads.make("llama2-13b", seed=args.seed, values_device="cpu", block_size=args.block_size)
    k8, v8, ks, vs = workloads.fp8_pools(w)
    k8, v8, ks, vs = k8.numpy(), v8.numpy(), ks.numpy(), vs.numpy()
    n = 8
    sub = workloads.subset(w, n)
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        oracle.paged_attention_fp8(w.q[:n], k8, v8, ks, vs, w.block_tables[:n], w.context_lens[:n], w.scale)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    value = round(decode_bytes(sub, kv_elem=1) / statistics.median(times) / 1e9, 4)
    return {
        "impl": "reference",
        "metric": "paged decode attn HBM GB/s on an FP8 (e4m3) pool & tokens*layers/s at 13B shape",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"llama2-13b with an FP8 pool, first {n} sequences", "block_size": w.block_size},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"first {n} of {w.num_seqs} sequences per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_blockmgr_reference(args, world):
    """The oracle's sequential append_slots on the host for the same decode step."""
    import oracle

    w = workloads.make("llama2-13b", seed=args.seed, values_device="cpu", block_size=args.block_size)
    B, bs = w.num_seqs, w.block_size
    mbs = (int(w.context_lens.max()) + args.steps + args.warmup + 2 * bs) // bs + 1
    st = oracle.bm_init(B * mbs + 64)
    ot = np.full((B, mbs), -1, np.int32)
    st, ot, oc, _, _, _ = oracle.bm_append_slots(st, ot, np.zeros(B, np.int32), w.context_lens.astype(np.int32), bs)
    ones = np.ones(B, np.int32)
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        st, ot, oc, _, _, _ = oracle.bm_append_slots(st, ot, oc, ones, bs)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    value = round(statistics.median(times) * 1e6, 3)
    return {
        "impl": "reference", "metric": "device block-manager append_slots microseconds per decode step",
        "value": value, "unit": "us", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 4), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "int32", "data": "synthetic",
        "config": {"workload": f"llama2-13b batch: {B} sequences, one new token each", "block_size": bs},
        "cpu_baseline": {"value": value, "unit": "us", "cores": 1, "kind": "oracle",
                         "sample": "the whole decode step per step"},
        "e2e": {"value": value, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: rank 0 times it on the host cores,
    one bounded sample of the workload per step."""
    if rank != 0:
        return None
    if args.workload in workloads.PREFILL_WORKLOADS:
        return run_prefill_reference(args, world)
    if args.workload in SWAP_WORKLOADS:
        return run_swap_reference(args, world)
    if args.workload in BM_WORKLOADS:
        return run_blockmgr_reference(args, world)
    if args.workload in FP8_WORKLOADS:
        return run_fp8_reference(args, world)
    w = workloads.make(args.workload, seed=args.seed, values_device="cpu", block_size=args.block_size)
    per_step_budget = max(0.05, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    pools = oracle_pools(w)
    for _ in range(args.warmup):
        cpu_baseline(w, per_step_budget, pools=pools)
    vals, tls = [], []
    t_all = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(w, per_step_budget, label="oracle", pools=pools)
        vals.append(last["value"])
        tls.append(last["tokens_layers_per_s"])
    t_all = time.perf_counter() - t_all
    value = statistics.median(vals)
    single = None
    if w.name in SINGLE_THREAD_WORKLOADS:  # outside the timed steps
        single = cpu_baseline(w, 0.05, pools=pools, single_thread_s=per_step_budget)["single_thread"]
    return {
        "impl": "reference",
        "metric": "paged decode attn HBM GB/s (% of B200 peak) & tokens·layers/s at 13B shape",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_all / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.description}", "block_size": w.block_size,
                   "num_seqs": w.num_seqs, "seed": args.seed},
        "tokens_layers_per_s": statistics.median(tls),
        "cpu_baseline": dict({"value": value, "unit": "GB/s", "cores": last["cores"], "kind": "oracle",
                              "sample": last["sample"]}, **({"single_thread": single} if single else {})),
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["pkv", "reference"], default="pkv")
    ap.add_argument("--workload", default="llama2-13b",
                    choices=list(workloads.WORKLOADS) + list(workloads.PREFILL_WORKLOADS) + list(SWAP_WORKLOADS)
                    + list(BM_WORKLOADS) + list(FP8_WORKLOADS))
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--partition-tokens", type=int, default=-1, help="-1: the workload's choice, 0: library's")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--max-seqs", type=int, default=0, help="time only the first N sequences (profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-shapes", action="store_true",
                    help="skip the decode-alone timings of the other shapes after the headline step")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1 and args.impl == "pkv":
        import datetime

        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        elif args.workload in workloads.PREFILL_WORKLOADS:
            line = run_prefill_cuda(args, rank, world, dist)
        elif args.workload in SWAP_WORKLOADS:
            line = run_swap_cuda(args, rank, world, dist)
        elif args.workload in BM_WORKLOADS:
            line = run_blockmgr_cuda(args, rank, world, dist)
        elif args.workload in FP8_WORKLOADS:
            line = run_fp8_cuda(args, rank, world, dist)
        else:
            line = run_cuda(args, rank, world, dist)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
