#!/usr/bin/env python
"""Throughput of exact attention (forward + backward) on B200 through libfa_sm100.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward (fa_fwd) and one backward (fa_bwd) pass over one batch of the
workload (default: GPT-style 2K causal self-attention, B=8, H=16, N=2048, d=128, bf16,
seeded i.i.d. N(0,1) inputs).  FLOPs follow the metric's convention: 4 B H N^2 d for the
forward, halved when causal, and 2.5x that for the backward; a local-attention workload
counts 4 d flop per visible (query, key) pair.

--workload varlen_32k_ragged times fa_fwd_varlen + fa_bwd_varlen over a packed batch of
ragged sequences (FLOPs of the visible pairs of each sequence); dropout_8k_causal times
the dropout forward and backward; blocksparse_8k_causal times the block-sparse forward and
backward (FLOPs of the pairs of the enabled blocks).

Decode workloads (--workload decode_*) time one fa_decode call per step (new query rows
against a resident key/value cache, split over the cache and merged); their metric is
the cache-read bandwidth in GB/s against the measured HBM copy peak.

The `e2e` leg runs the same steps through the public binding with each step's inputs copied
from pinned host memory and its results copied back, overlapped across neighbouring steps
on three streams (input copy, kernels, result copy) with two device buffer sets.

Rank 0 prints one JSON line.  Under torchrun each rank (one GPU each) processes its own
shard of a global batch of N x B sequences with the unchanged kernels (no collective on
the data path); the timed region is bracketed by barriers and the slowest rank's time is
used, so `value` is the whole job's TFLOP/s ("scaling": "weak").

`--impl reference` times the fp64 CPU oracle (the parity reference) on a bounded sample of
the same workload on this host's cores, on rank 0 only.
"""
from __future__ import annotations

import argparse
import csv
import datetime as _dt
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd+bwd TFLOP/s at 1 B200 and % of dense-BF16 tensor peak"
E2E_OVERLAP = ("each step's inputs host->device, its kernels and its results device->host on three "
               "streams, overlapping neighbouring steps, with two device buffer sets")
UNIT = "TFLOP/s"
NOMINAL_BF16_TFLOPS = 2250.0  # NVIDIA's dense bf16 figure for one B200, for context only
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu capture
    (profiles/dram_traffic.json), or None when there is none or a source file of the
    kernel has changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            entries = json.load(f)["entries"]
        for e in entries:
            if e["kernel"] != kernel or e["workload"] != workload:
                continue
            for src, digest in zip(e["sources"], e["sources_sha256"]):
                with open(os.path.join(ROOT, src), "rb") as f:
                    if hashlib.sha256(f.read()).hexdigest() != digest:
                        return None
            return int(e["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        return None
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, kept only inside [t0, t1]."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        self.t0 = _dt.datetime.now()

    def stop(self):
        self.t1 = _dt.datetime.now()
        time.sleep(0.12)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        self.file.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.file.read())) if len(r) >= 9]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons, n = [], [], set(), 0
        for r in rows:
            try:
                ts = _dt.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                continue
            if self.t0 and self.t1 and not (self.t0 <= ts <= self.t1):
                continue
            n += 1
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                pass
            for name, val in zip(names, r[5:9]):
                if val.strip() == "Active":
                    reasons.add(name)
        os.unlink(self.file.name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": n}


def _oracle_sample(w, heads: int, seed: int):
    """fp64 oracle fwd+bwd on the first `heads` query heads (whole K/V groups) of batch
    row 0 of the workload's inputs; returns (seconds, metric FLOPs of the sample)."""
    import numpy as np
    import torch
    import oracle
    from exact_io_aware_83_b200.inputs import draw
    g = w.Hq // w.Hkv
    groups = max(1, heads // g)
    q, k, v, do = draw(1, groups * g, groups, w.N, w.d, seed, w.q_std)
    f64 = lambda t: t.float().double().numpy()
    q, k, v, do = f64(q), f64(k), f64(v), f64(do)
    bm = w.block_mask()
    if bm is not None:
        bm = bm[:1, :groups * g].contiguous()
    t0 = time.perf_counter()
    if bm is not None:
        oracle.attention_fwd_blocksparse(q, k, v, bm.numpy(), w.causal, w.scale)
        if w.backward:
            oracle.attention_bwd_blocksparse(q, k, v, do, bm.numpy(), w.causal, w.scale)
    elif w.dropout_p:
        oracle.attention_fwd_dropout(q, k, v, w.causal, w.scale, w.dropout_p, w.dropout_seed)
        if w.backward:
            oracle.attention_bwd_dropout(q, k, v, do, w.causal, w.scale, w.dropout_p, w.dropout_seed)
    elif w.window is not None:
        oracle.attention_fwd_window(q, k, v, w.window[0], w.window[1], w.scale)
        if w.backward:
            oracle.attention_bwd_window(q, k, v, do, w.window[0], w.window[1], w.scale)
    else:
        oracle.attention_fwd(q, k, v, w.causal, w.scale)
        if w.backward:
            oracle.attention_bwd(q, k, v, do, w.causal, w.scale)
    dt = time.perf_counter() - t0
    flops = (w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)) * (groups * g) / (w.B * w.Hq)
    if bm is not None:  # the sampled heads' own mask
        from exact_io_aware_83_b200.inputs import blocksparse_pairs
        flops = 4.0 * blocksparse_pairs(bm, w.N, w.causal) * w.d * (3.5 if w.backward else 1.0)
    return dt, flops


def _e2e_pipelined(host_in, dev_in, dev_out, host_out, compute, n_steps, n_warm, barrier):
    """End-to-end time (ms) of `n_steps` steps through the public API, every step copying its
    inputs from pinned host memory to the device and its results back.  Two sets of device
    buffers alternate, and three streams overlap step i's input copy, step i-1's kernels and
    step i-2's result copy (as a training loop prefetches its next batch); events order the
    reuse of each buffer set.  host_in: pinned inputs (one set, re-sent every step);
    dev_in / dev_out / host_out: two sets each; compute(slot) launches one step's kernels on
    the current stream over set `slot`."""
    import torch
    h2d, comp, d2h = (torch.cuda.Stream() for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        sl = i % 2
        if i >= 2:
            h2d.wait_event(ev_done[sl])        # step i-2's kernels have read this input set
        with torch.cuda.stream(h2d):
            for dev, hst in zip(dev_in[sl], host_in):
                dev.copy_(hst, non_blocking=True)
            ev_in[sl].record(h2d)
        comp.wait_event(ev_in[sl])
        if i >= 2:
            comp.wait_event(ev_out[sl])        # step i-2's results have left this output set
        with torch.cuda.stream(comp):
            compute(sl)
            ev_done[sl].record(comp)
        d2h.wait_event(ev_done[sl])
        with torch.cuda.stream(d2h):
            for hst, dev in zip(host_out[sl], dev_out[sl]):
                hst.copy_(dev, non_blocking=True)
            ev_out[sl].record(d2h)

    for i in range(n_warm):
        one(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    for i in range(n_steps):
        one(i)
    # the last result copy ends the region; wait for every stream
    d2h.wait_stream(h2d)
    d2h.wait_stream(comp)
    e1.record(d2h)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1)


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    cores = _cores()
    oracle.set_threads(cores)
    # Size the per-step sample so the whole run stays near a two-minute budget: whole
    # K/V-head groups of batch row 0, at least one.
    g = w.Hq // w.Hkv
    t_group, _ = _oracle_sample(w, g, w.seed)
    budget = 120.0 / (args.steps + args.warmup)
    heads = g * max(1, min(w.Hkv, int(budget // max(t_group, 1e-6))))
    for _ in range(args.warmup):
        _oracle_sample(w, heads, w.seed)
    total_t, total_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = _oracle_sample(w, heads, w.seed)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    sample = (f"batch row 0, query heads 0..{heads - 1} of {w.name} (fwd"
              f"{'+bwd' if w.backward else ''}), fp64 oracle, per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(w, world):
    if hasattr(w, "Nk"):
        return {"workload": w.name, "B_per_gpu": w.B, "global_batch": w.B * world, "Hq": w.Hq,
                "Hkv": w.Hkv, "new_tokens": w.Nq, "cache_len": w.Nk, "head_dim": w.d,
                "causal": w.causal, "passes": "decode", "parallelism": f"dp{world}",
                "l2": f"cache exceeds L2 ({w.cache_bytes() / 1e6:.0f} MB vs 126 MB); no flush"}
    c = {"workload": w.name, "B_per_gpu": w.B, "global_batch": w.B * world, "Hq": w.Hq,
         "Hkv": w.Hkv, "seq_len": w.N, "head_dim": w.d, "causal": w.causal,
         "passes": "fwd+bwd" if w.backward else "fwd", "parallelism": f"dp{world}",
         "l2": "inputs exceed L2 (q, k, v, dO = "
               f"{4 * w.B * w.Hq * w.N * w.d * 2 / 1e6:.0f} MB vs 126 MB); no flush"}
    if w.window is not None:
        c["window"] = list(w.window)
    if w.dropout_p:
        c["dropout_p"] = w.dropout_p
        c["dropout_seed"] = w.dropout_seed
    if w.block_density:
        c["block_mask"] = {"block": 128, "density": w.block_density, "diagonal": True,
                           "mask_seed": w.mask_seed,
                           "enabled_pairs_share_of_causal": round(
                               w.fwd_flops() / (2.0 * w.B * w.Hq * w.N * w.N * w.d), 4)}
    return c


def _config_varlen(w, world):
    lens = w.lens()
    return {"workload": w.name, "sequences_per_gpu": w.n_seqs, "tokens_per_gpu": sum(lens),
            "longest": max(lens), "mean_len": w.mean_len, "Hq": w.H, "Hkv": w.H, "head_dim": w.d,
            "causal": w.causal, "passes": "fwd+bwd", "parallelism": f"dp{world}",
            "l2": f"inputs exceed L2 (q, k, v, dO = {4 * sum(lens) * w.H * w.d * 2 / 1e6:.0f} MB vs "
                  "126 MB); no flush"}


def _oracle_varlen_sample(w, n_seqs: int):
    """fp64 oracle fwd+bwd on the n_seqs shortest sequences; returns (seconds, FLOPs)."""
    import oracle
    from exact_io_aware_83_b200.inputs import draw_packed
    lens = sorted(w.lens())[:n_seqs]
    q, k, v, do, cq, ck = draw_packed(lens, lens, w.H, w.H, w.d, w.seed)
    f64 = lambda t: t.float().double().numpy()
    right = 0 if w.causal else -1
    t0 = time.perf_counter()
    oracle.attention_fwd_varlen(f64(q), f64(k), f64(v), cq.numpy(), ck.numpy(), -1, right, w.scale)
    oracle.attention_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cq.numpy(), ck.numpy(), -1, right,
                                w.scale)
    dt = time.perf_counter() - t0
    pairs = sum(L * (L + 1) // 2 if w.causal else L * L for L in lens)
    return dt, 3.5 * 4.0 * w.H * w.d * pairs


def run_reference_varlen(args, w):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    cores = _cores()
    oracle.set_threads(cores)
    t1, f1 = _oracle_varlen_sample(w, 1)
    budget = 120.0 / (args.steps + args.warmup)
    # Add the next-shortest sequences while the estimated time (proportional to the
    # visible pairs, i.e. to the FLOPs) stays within the per-step budget.
    per_flop = t1 / f1
    lens = sorted(w.lens())
    n, cost = 0, 0.0
    for L in lens:
        f = 3.5 * 4.0 * w.H * w.d * (L * (L + 1) // 2 if w.causal else L * L)
        if n > 0 and cost + f * per_flop > budget:
            break
        n, cost = n + 1, cost + f * per_flop
    for _ in range(args.warmup):
        _oracle_varlen_sample(w, n)
    tt, tf = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = _oracle_varlen_sample(w, n)
        tt += dt
        tf += fl
    value = tf / tt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config_varlen(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"the {n} shortest sequences of {w.name}, fp64 oracle fwd+bwd, per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours_varlen(args, w):
    import torch
    import torch.distributed as dist
    from exact_io_aware_83_b200 import fa
    from exact_io_aware_83_b200.inputs import draw_packed
    from exact_io_aware_83_b200.shard import max_over_ranks, rank_seed

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    fa.load()
    lens = w.lens()
    host = draw_packed(lens, lens, w.H, w.H, w.d, rank_seed(w.seed, rank))
    q, k, v, do, cq, ck = (t.cuda() for t in host)
    mx = max(lens)
    o = torch.empty_like(q)
    lse = torch.empty((q.shape[0], w.H), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_varlen_workspace_bytes(w.H, q.shape[0], w.d), dtype=torch.uint8,
                     device="cuda")

    def step():
        fa.fwd_varlen(q, k, v, cq, ck, mx, mx, causal=w.causal, scale=w.scale, out=o, lse=lse)
        fa.bwd_varlen(q, k, v, o, lse, do, cq, ck, mx, mx, causal=w.causal, scale=w.scale,
                      workspace=ws, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_device_status(None) != fa.FA_OK:
        raise SystemExit("device status not clean after warm-up")
    sampler = ClockSampler(local)
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    fa.fa_kernel_timing(True)
    sampler.start()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    fa.fa_kernel_timing(False)
    ms = max_over_ranks(e0.elapsed_time(e1))
    fwd_ms, nfwd = fa.fa_kernel_time_ms(0)
    bwd_ms, nbwd = fa.fa_kernel_time_ms(1)
    if fa.fa_device_status(None) != fa.FA_OK:
        raise SystemExit("device status not clean after the timed region")
    clocks = sampler.summary()
    step_flops = w.fwd_flops() + w.bwd_flops()
    value = step_flops * args.steps * world / (ms / 1e3) / 1e12

    pin = lambda t: t.pin_memory()
    host_in = [pin(t) for t in host[:4]]
    outs = [o, lse, dq, dk, dv]
    dev_in = [[q, k, v, do], [torch.empty_like(t) for t in (q, k, v, do)]]
    dev_out = [outs, [torch.empty_like(t) for t in outs]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs] for _ in range(2)]

    def compute(sl):
        qq, kk, vv, dd = dev_in[sl]
        oo, ll, gq, gk, gv = dev_out[sl]
        fa.fwd_varlen(qq, kk, vv, cq, ck, mx, mx, causal=w.causal, scale=w.scale, out=oo, lse=ll)
        fa.bwd_varlen(qq, kk, vv, oo, ll, dd, cq, ck, mx, mx, causal=w.causal, scale=w.scale,
                      workspace=ws, dq=gq, dk=gk, dv=gv)

    e2e_steps = max(8, args.steps // 10)
    e2e_ms = max_over_ranks(_e2e_pipelined(host_in, dev_in, dev_out, host_out, compute, e2e_steps, 2,
                                           barrier))
    nb = lambda *ts: sum(t.numel() * t.element_size() for t in ts)

    peaks, peak_src = _peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = w.bwd_flops() / (bwd_ms / nbwd / 1e3) / 1e12
    kernels = {
        "fa_fwd_kernel": {"ms_per_launch": fwd_ms / nfwd, "tflops": w.fwd_flops() / (fwd_ms / nfwd / 1e3) / 1e12},
        "fa_bwd_main_kernel": {"ms_per_launch": bwd_ms / nbwd, "tflops": achieved},
    }
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config_varlen(w, world),
        "frac_of_peak": value / world / peak,
        "roofline": {"bound": "tensor", "kernel": "fa_bwd_main_kernel", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": _profile_traffic("fa_bwd_main_kernel", w.name),
                     "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"},
        "kernels": kernels,
        "e2e": {"value": step_flops * e2e_steps * world / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": nb(q, k, v, do), "d2h_bytes_per_step": nb(o, lse, dq, dk, dv),
                "steps": e2e_steps, "overlap": E2E_OVERLAP},
        "gpu_launches": args.steps * 4,
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        import oracle
        cores = _cores()
        oracle.set_threads(cores)
        dt, fl = _oracle_varlen_sample(w, 2)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"the 2 shortest sequences of {w.name}, fp64 oracle fwd+bwd, one pass, {dt:.1f} s wall"}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    from exact_io_aware_83_b200 import fa
    from exact_io_aware_83_b200.inputs import draw
    from exact_io_aware_83_b200.shard import max_over_ranks, rank_seed

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    fa.load()
    qh, kh, vh, doh = draw(w.B, w.Hq, w.Hkv, w.N, w.d, rank_seed(w.seed, rank), w.q_std)
    q, k, v, do = (t.cuda() for t in (qh, kh, vh, doh))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8,
                     device="cuda")
    bmh = w.block_mask()
    bmd = None if bmh is None else bmh.cuda()

    def run(q, k, v, do, o, lse, dq, dk, dv, bm):
        fa.fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, window=w.window,
               dropout_p=w.dropout_p, seed=w.dropout_seed, block_mask=bm)
        if w.backward:
            fa.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, workspace=ws, dq=dq,
                   dk=dk, dv=dv, window=w.window, dropout_p=w.dropout_p, seed=w.dropout_seed,
                   block_mask=bm)

    def step():
        run(q, k, v, do, o, lse, dq, dk, dv, bmd)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_device_status(None) != fa.FA_OK:
        raise SystemExit("device status not clean after warm-up")

    sampler = ClockSampler(local)
    time.sleep(0.3)  # let nvidia-smi start sampling
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    fa.fa_kernel_timing(True)
    sampler.start()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    fa.fa_kernel_timing(False)
    ms_local = e0.elapsed_time(e1)
    ms = max_over_ranks(ms_local)
    fwd_ms, nfwd = fa.fa_kernel_time_ms(0)
    bwd_ms, nbwd = fa.fa_kernel_time_ms(1)
    status = fa.fa_device_status(None)
    if status != fa.FA_OK:
        raise SystemExit(f"device status {status} after the timed region")
    clocks = sampler.summary()

    step_flops = w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)
    value = step_flops * args.steps * world / (ms / 1e3) / 1e12

    # ---- end to end through the public API: pinned host inputs in, results back to host
    pin = lambda t: t.pin_memory()
    ins = [qh, kh, vh] + ([doh] if w.backward else []) + ([] if bmh is None else [bmh])
    host_in = [pin(t) for t in ins]
    outs = [o, lse] + ([dq, dk, dv] if w.backward else [])
    dev_in = [[q, k, v] + ([do] if w.backward else []) + ([] if bmd is None else [bmd]),
              [torch.empty_like(t, device="cuda") for t in ins]]
    dev_out = [outs, [torch.empty_like(t) for t in outs]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs] for _ in range(2)]

    def compute(sl):
        di, do_ = dev_in[sl], dev_out[sl]
        qq, kk, vv = di[0], di[1], di[2]
        dd = di[3] if w.backward else None
        bm = di[-1] if bmd is not None else None
        if w.backward:
            run(qq, kk, vv, dd, do_[0], do_[1], do_[2], do_[3], do_[4], bm)
        else:
            run(qq, kk, vv, None, do_[0], do_[1], None, None, None, bm)

    e2e_steps = max(8, args.steps // 10)
    e2e_ms = max_over_ranks(_e2e_pipelined(host_in, dev_in, dev_out, host_out, compute, e2e_steps, 2,
                                           barrier))
    nbytes = lambda *ts: sum(t.numel() * t.element_size() for t in ts)
    h2d = nbytes(*dev_in[0])
    d2h = nbytes(*outs)
    e2e_value = step_flops * e2e_steps * world / (e2e_ms / 1e3) / 1e12

    peaks, peak_src = _peaks()
    # Dominant kernel: the backward main kernel (or the forward when there is no backward).
    if w.backward and nbwd:
        dom_name, dom_ms, dom_n, dom_flops = "fa_bwd_main_kernel", bwd_ms, nbwd, w.bwd_flops()
    else:
        dom_name, dom_ms, dom_n, dom_flops = "fa_fwd_kernel", fwd_ms, nfwd, w.fwd_flops()
    achieved = dom_flops / (dom_ms / dom_n / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = _profile_traffic(dom_name, w.name)
    kernels = {}
    if nfwd:
        kernels["fa_fwd_kernel"] = {"ms_per_launch": fwd_ms / nfwd,
                                    "tflops": w.fwd_flops() / (fwd_ms / nfwd / 1e3) / 1e12}
    if nbwd:
        kernels["fa_bwd_main_kernel"] = {"ms_per_launch": bwd_ms / nbwd,
                                         "tflops": w.bwd_flops() / (bwd_ms / nbwd / 1e3) / 1e12}
    for kname, kd in kernels.items():
        kd["frac_of_burst_peak"] = kd["tflops"] / peak
        kd["frac_of_sustained_peak"] = kd["tflops"] / float(peaks["bf16_tflops_sustained"])
        kd["frac_of_nominal_peak"] = kd["tflops"] / NOMINAL_BF16_TFLOPS

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w, world),
        "frac_of_peak": value / world / peak,
        "roofline": {"bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "overlap": E2E_OVERLAP},
        "gpu_launches": args.steps * (1 + (3 if w.backward else 0)),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        import oracle
        cores = _cores()
        oracle.set_threads(cores)
        heads = max(1, min(w.Hq, args.sample_heads))
        dt, fl = _oracle_sample(w, heads, w.seed)
        line["cpu_baseline"] = {
            "value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"batch row 0, query heads 0..{heads - 1} of {w.name}, fp64 oracle "
                      f"fwd{'+bwd' if w.backward else ''}, one pass, {dt:.1f} s wall"}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


DECODE_METRIC = "decode KV-cache read bandwidth GB/s at 1 B200 and % of measured HBM copy peak"


def _oracle_decode_sample(w, groups: int):
    """fp64 oracle decode of the first `groups` K/V-head groups of batch row 0; returns
    (seconds, algorithmic bytes of the sample)."""
    import oracle
    from exact_io_aware_83_b200.inputs import draw_decode
    g = w.Hq // w.Hkv
    q, k, v = draw_decode(1, groups * g, groups, w.Nq, w.Nk, w.d, w.seed)
    f64 = lambda t: t.float().double().numpy()
    q, k, v = f64(q), f64(k), f64(v)
    t0 = time.perf_counter()
    oracle.attention_decode(q, k, v, None, w.causal, w.scale)
    dt = time.perf_counter() - t0
    return dt, w.io_bytes() * groups / (w.B * w.Hkv)


def run_reference_decode(args, w):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    cores = _cores()
    oracle.set_threads(cores)
    t1, _ = _oracle_decode_sample(w, 1)
    budget = 120.0 / (args.steps + args.warmup)
    groups = max(1, min(w.B * w.Hkv if w.B == 1 else w.Hkv, int(budget // max(t1, 1e-6))))
    for _ in range(args.warmup):
        _oracle_decode_sample(w, groups)
    tt, tb = 0.0, 0.0
    for _ in range(args.steps):
        dt, nb = _oracle_decode_sample(w, groups)
        tt += dt
        tb += nb
    value = tb / tt / 1e9
    line = {
        "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": _config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"batch row 0, K/V heads 0..{groups - 1} of {w.name}, fp64 oracle, per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours_decode(args, w):
    import torch
    import torch.distributed as dist
    from exact_io_aware_83_b200 import fa
    from exact_io_aware_83_b200.inputs import draw_decode
    from exact_io_aware_83_b200.shard import max_over_ranks, rank_seed

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    fa.load()
    qh, kh, vh = draw_decode(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, rank_seed(w.seed, rank))
    q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
    del kh, vh
    S = fa.fa_decode_num_splits(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)
    ws = torch.empty(max(16, fa.fa_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, S)),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device="cuda")

    def step():
        fa.decode(q, k, v, causal=w.causal, scale=w.scale, num_splits=S, out=o, lse=lse,
                  workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_device_status(None) != fa.FA_OK:
        raise SystemExit("device status not clean after warm-up")
    sampler = ClockSampler(local)
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    fa.fa_kernel_timing(True)
    sampler.start()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    sampler.stop()
    fa.fa_kernel_timing(False)
    ms = max_over_ranks(e0.elapsed_time(e1))
    dec_ms, ndec = fa.fa_kernel_time_ms(2)
    if fa.fa_device_status(None) != fa.FA_OK:
        raise SystemExit("device status not clean after the timed region")
    clocks = sampler.summary()
    value = w.io_bytes() * args.steps * world / (ms / 1e3) / 1e9

    # End to end: the new query rows come from pinned host memory and O, LSE go back; the
    # cache stays resident on the device, as it does between decode steps.
    host_in = [qh.pin_memory()]
    dev_in = [[q], [torch.empty_like(q)]]
    dev_out = [[o, lse], [torch.empty_like(o), torch.empty_like(lse)]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, lse)] for _ in range(2)]

    def compute(sl):
        fa.decode(dev_in[sl][0], k, v, causal=w.causal, scale=w.scale, num_splits=S,
                  out=dev_out[sl][0], lse=dev_out[sl][1], workspace=ws)

    e2e_steps = max(8, args.steps // 10)
    e2e_ms = max_over_ranks(_e2e_pipelined(host_in, dev_in, dev_out, host_out, compute, e2e_steps, 2,
                                           barrier))
    nb = lambda *ts: sum(t.numel() * t.element_size() for t in ts)

    peaks, peak_src = _peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = w.io_bytes() / (dec_ms / ndec / 1e3) / 1e9
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict(_config(w, world), num_splits=S),
        "frac_of_peak": value / world / peak,
        "roofline": {"bound": "hbm", "kernel": "fa_decode_kernel", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": _profile_traffic("fa_decode_kernel", w.name),
                     "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json hbm_gbs)"},
        "e2e": {"value": w.io_bytes() * e2e_steps * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": nb(q), "d2h_bytes_per_step": nb(o, lse), "steps": e2e_steps,
                "overlap": E2E_OVERLAP},
        "gpu_launches": args.steps * (2 if S > 1 else 1),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        import oracle
        cores = _cores()
        oracle.set_threads(cores)
        dt, nbytes = _oracle_decode_sample(w, 1)
        line["cpu_baseline"] = {
            "value": nbytes / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"batch row 0, K/V head 0 of {w.name}, fp64 oracle decode, one pass, {dt:.2f} s wall"}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gpt_2k_causal")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--sample-heads", type=int, default=4,
                    help="query heads in the oracle's bounded CPU sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    from exact_io_aware_83_b200.inputs import DECODE_WORKLOADS, VARLEN_WORKLOADS, WORKLOADS
    if args.workload in VARLEN_WORKLOADS:
        w = VARLEN_WORKLOADS[args.workload]
        if args.impl == "reference":
            return run_reference_varlen(args, w)
        return run_ours_varlen(args, w)
    if args.workload in DECODE_WORKLOADS:
        w = DECODE_WORKLOADS[args.workload]
        if args.impl == "reference":
            return run_reference_decode(args, w)
        return run_ours_decode(args, w)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
