#!/usr/bin/env python
"""Throughput of exact attention (forward + backward) on B200 through libfa_sm100.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--scaling weak|strong]

A step is one forward (fa_fwd) and one backward (fa_bwd) pass over one batch of the
workload (default: long-context causal self-attention, B=2, H=16, N=8192, d=128, bf16,
seeded i.i.d. N(0,1) inputs - the largest single-GPU workload, the pages' 8K-context
rows).  FLOPs follow the metric's convention: 4 B H N^2 d for the forward, halved when
causal, and 2.5x that for the backward; a local-attention workload counts 4 d flop per
visible (query, key) pair.  Each kernel is also reported against its two bounds: the
tensor-core time of its FLOPs at the measured bf16 peak, and the MUFU time of its
exponentials (one per visible score and pass) at 16 per clock per SM.

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

Rank 0 prints one JSON line.  Under torchrun each rank (one GPU each) runs the unchanged
kernels on its own share with no collective on the data path; the timed region is
bracketed by barriers and the slowest rank's time is used, so `value` is the whole job's
TFLOP/s.  --scaling weak (default): each rank processes its own batch of the workload's
shape, a global batch of N x B sequences.  --scaling strong: the workload itself is split
by (batch row, K/V head) groups, so B = 2 at 8K context still spreads over 32 ranks.

The CPU baseline times the fp64 oracle (the parity reference, built -O3 -march=native for
the host) on whole K/V-head groups of the workload, one oracle call per group, for about
--cpu-budget seconds, and extrapolates the full workload's time from it.
`--impl reference` times the same oracle on a per-step sample of the same workload, on
rank 0 only.
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


# The library takes 128-query backward steps for dense d = 128 attention from this sequence
# length on (kQ128MinN in exact_io_aware_83_b200/csrc/fa_bwd.cuh).
Q128_MIN_N = 4096


def _bwd_kernel_name(w) -> str:
    """The backward main kernel the library's dispatch runs for workload `w`: dense
    attention without dropout runs as CTA pairs at d = 256 and with 128-query steps at
    d = 128 from Q128_MIN_N on; everything else runs fa_bwd_main_kernel."""
    plain = w.block_density == 0 and w.window is None and not w.dropout_p
    if plain and w.d == 256:
        return "fa_bwd_pair_kernel"
    if plain and w.d == 128 and w.N >= Q128_MIN_N:
        return "fa_bwd_q128_kernel"
    return "fa_bwd_main_kernel"


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
    """SM clock, power and clock-event (throttle) reasons sampled DURING the timed region.

    A thread polls NVML (read-only queries) every `period_s` between start() and stop(),
    so even a timed region of a few tens of milliseconds gets samples; where NVML is
    unavailable it falls back to `nvidia-smi -lms 20`, whose samples are kept only when
    their timestamps fall inside the region."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        import threading
        self.period = period_s
        self.samples = []          # (sm_mhz, max_mhz, power_w, reason bits)
        self.source = "nvml"
        self.nvml = None
        self.handle = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(gpu_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus.encode())
            except Exception:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.nvml = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
            self.source = "nvidia-smi"
        self._smi = None if self.nvml is not None else _SmiSampler(gpu_index)

    def _poll(self):
        nv, h = self.nvml, self.handle
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                bits = int(get_reasons(h)) if get_reasons else 0
                self.samples.append((sm, self.max_mhz, pw, bits))
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.nvml is None:
            self._smi.start()
            return
        import threading
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()

    def stop(self):
        if self.nvml is None:
            self._smi.stop()
            return
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if self.nvml is None:
            return self._smi.summary()
        sm = [x[0] for x in self.samples]
        reasons = set()
        for _, _, _, bits in self.samples:
            for name, const in self.REASONS:
                if bits & int(getattr(self.nvml, const, 0)):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(sm) if sm else None,
                "power_w_max": max(x[2] for x in self.samples) if self.samples else None,
                "reasons": sorted(reasons), "samples": len(self.samples),
                "source": f"NVML every {self.period * 1e3:.0f} ms during the timed region"}


class _SmiSampler:
    """nvidia-smi clock / throttle-reason samples, kept only inside [t0, t1]."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)  # let nvidia-smi start sampling
        self.t0 = self.t1 = None

    def start(self):
        self.t0 = _dt.datetime.now()

    def stop(self):
        self.t1 = _dt.datetime.now()
        time.sleep(0.05)
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
                "reasons": sorted(reasons), "samples": n,
                "source": "nvidia-smi -lms 20 during the timed region"}


def _oracle_groups(w, n_groups: int, seed: int, budget_s: float | None = None):
    """Time the fp64 oracle (fwd, plus bwd when the workload has one) on whole K/V-head
    groups of batch row 0 of the workload's shapes, one oracle call per group, so the
    working set and the per-flop rate do not depend on how many groups are sampled.
    Stops after `n_groups` groups, or earlier once `budget_s` seconds of oracle time have
    been spent (at least one group).  Returns (seconds, metric FLOPs, groups timed)."""
    import oracle
    from exact_io_aware_83_b200.inputs import draw
    g = w.Hq // w.Hkv
    n_groups = max(1, min(n_groups, w.Hkv))
    q, k, v, do = draw(1, n_groups * g, n_groups, w.N, w.d, seed, w.q_std)
    f64 = lambda t: t.float().double().numpy()
    bm = w.block_mask()
    total_t, groups = 0.0, 0
    for kv in range(n_groups):
        qs, ks, vs, ds = (f64(t[:, kv * g:(kv + 1) * g] if t.shape[1] == n_groups * g else t[:, kv:kv + 1])
                          for t in (q, k, v, do))
        t0 = time.perf_counter()
        if bm is not None:
            m = bm[:1, kv * g:(kv + 1) * g].contiguous().numpy()
            oracle.attention_fwd_blocksparse(qs, ks, vs, m, w.causal, w.scale)
            if w.backward:
                oracle.attention_bwd_blocksparse(qs, ks, vs, ds, m, w.causal, w.scale)
        elif w.dropout_p:
            oracle.attention_fwd_dropout(qs, ks, vs, w.causal, w.scale, w.dropout_p, w.dropout_seed)
            if w.backward:
                oracle.attention_bwd_dropout(qs, ks, vs, ds, w.causal, w.scale, w.dropout_p, w.dropout_seed)
        elif w.window is not None:
            oracle.attention_fwd_window(qs, ks, vs, w.window[0], w.window[1], w.scale)
            if w.backward:
                oracle.attention_bwd_window(qs, ks, vs, ds, w.window[0], w.window[1], w.scale)
        else:
            oracle.attention_fwd(qs, ks, vs, w.causal, w.scale)
            if w.backward:
                oracle.attention_bwd(qs, ks, vs, ds, w.causal, w.scale)
        total_t += time.perf_counter() - t0
        groups += 1
        if budget_s is not None and total_t >= budget_s:
            break
    per_group = (w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)) / (w.B * w.Hkv)
    flops = per_group * groups
    if bm is not None:  # the sampled heads' own mask
        from exact_io_aware_83_b200.inputs import blocksparse_pairs
        flops = 4.0 * blocksparse_pairs(bm[:1, :groups * g].contiguous(), w.N, w.causal) * w.d * (
            3.5 if w.backward else 1.0)
    return total_t, flops, groups


def _cpu_baseline_line(w, seconds, flops, groups, cores, note):
    """The cpu_baseline object: the oracle's rate on the sample, what the sample was, and
    the full workload's time extrapolated from it (per group; groups are independent)."""
    import oracle
    from oracle import build as oracle_build
    return {"value": flops / seconds / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": oracle_build.cpu_model(), "build": oracle.build_flags(),
            "sample": (f"K/V-head groups 0..{groups - 1} of batch row 0 of {w.name} ({groups * (w.Hq // w.Hkv)} "
                       f"query heads), fp64 oracle fwd{'+bwd' if w.backward else ''}, one oracle call per "
                       f"group, {seconds:.1f} s {note}"),
            "full_size_s_extrapolated": seconds / groups * w.B * w.Hkv}


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
    oracle.use_build("native")
    cores = _cores()
    oracle.set_threads(cores)
    # Size the per-step sample so the whole run stays near a two-and-a-half-minute budget:
    # whole K/V-head groups of batch row 0, at least one.
    t_group, _, _ = _oracle_groups(w, 1, w.seed)
    budget = 150.0 / (args.steps + args.warmup)
    groups = max(1, min(w.Hkv, int(budget // max(t_group, 1e-6))))
    for _ in range(args.warmup):
        _oracle_groups(w, groups, w.seed)
    total_t, total_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl, _ = _oracle_groups(w, groups, w.seed)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    cpu = _cpu_baseline_line(w, total_t / args.steps, total_f / args.steps, groups, cores, "per step")
    cpu["value"] = value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, args.gpus),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _l2_note(nbytes: int) -> str:
    """How the timed region stands to the 126 MB L2: inputs larger than L2 need no flush."""
    if nbytes > 126e6:
        return f"inputs exceed L2 ({nbytes / 1e6:.0f} MB vs 126 MB); no flush"
    return (f"inputs fit in L2 ({nbytes / 1e6:.2f} MB vs 126 MB) and are not flushed: a parity-size "
            "workload, not a throughput line")


def _config(w, world):
    if hasattr(w, "Nk"):
        return {"workload": w.name, "B_per_gpu": w.B, "global_batch": w.B * world, "Hq": w.Hq,
                "Hkv": w.Hkv, "new_tokens": w.Nq, "cache_len": w.Nk, "head_dim": w.d,
                "causal": w.causal, "passes": "decode", "parallelism": f"dp{world}",
                "l2": f"cache exceeds L2 ({w.cache_bytes() / 1e6:.0f} MB vs 126 MB); no flush"}
    c = {"workload": w.name, "B_per_gpu": w.B, "global_batch": w.B * world, "Hq": w.Hq,
         "Hkv": w.Hkv, "seq_len": w.N, "head_dim": w.d, "causal": w.causal,
         "passes": "fwd+bwd" if w.backward else "fwd", "parallelism": f"dp{world}",
         "l2": _l2_note(((2 if w.backward else 1) * w.Hq + 2 * w.Hkv) * w.B * w.N * w.d * 2)}
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
    oracle.use_build("native")
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
        oracle.use_build("native")
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


def _parts(w, world: int, rank: int, scaling: str):
    """This rank's share of the work as (host tensors, block mask, batch rows, query heads,
    K/V heads) parts.  Weak scaling: one part, the whole workload drawn with the rank's own
    seed.  Strong scaling: the workload itself (one seed on every rank) split by
    (batch row, K/V head) groups, one part per contiguous segment of this rank's groups."""
    from exact_io_aware_83_b200.inputs import draw
    from exact_io_aware_83_b200.shard import rank_seed, segment_slices, shard_groups
    bmh = w.block_mask()
    if scaling == "weak":
        host = draw(w.B, w.Hq, w.Hkv, w.N, w.d, rank_seed(w.seed, rank), w.q_std)
        return [(host, bmh, w.B, w.Hq, w.Hkv)]
    full = draw(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, w.q_std)
    g = w.Hq // w.Hkv
    parts = []
    for seg in shard_groups(w.B, w.Hkv, world, rank):
        qh_, kvh_, bs = segment_slices(seg, g)
        host = tuple(t[bs, qh_ if t.shape[1] == w.Hq else kvh_].contiguous() for t in full)
        bm = None if bmh is None else bmh[bs, qh_].contiguous()
        parts.append((host, bm, seg.b_hi - seg.b_lo, (seg.kv_hi - seg.kv_lo) * g, seg.kv_hi - seg.kv_lo))
    return parts


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    from exact_io_aware_83_b200 import fa
    from exact_io_aware_83_b200.shard import max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.scaling == "strong" and w.dropout_p:
        raise SystemExit("--scaling strong: the dropout mask is a function of the global head "
                         "index, so a split problem would draw a different mask")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    fa.load()
    # Per part: device inputs [q, k, v, (dO), (mask)] and outputs [o, lse, (dq, dk, dv)],
    # one backward workspace per part.
    parts = []
    for host, bmh, B, Hq, Hkv in _parts(w, world, rank, args.scaling):
        ins = list(host[:3]) + ([host[3]] if w.backward else []) + ([] if bmh is None else [bmh])
        dev = [t.cuda() for t in ins]
        q = dev[0]
        outs = [torch.empty_like(q), torch.empty((B, Hq, w.N), dtype=torch.float32, device="cuda")]
        if w.backward:
            outs += [torch.empty_like(q), torch.empty_like(dev[1]), torch.empty_like(dev[2])]
        ws = torch.empty(fa.fa_bwd_workspace_bytes(B, Hq, Hkv, w.N, w.d), dtype=torch.uint8, device="cuda")
        parts.append({"host": ins, "dev": dev, "outs": outs, "ws": ws, "mask": bmh is not None})

    def run(part, dev, outs):
        q, k, v = dev[0], dev[1], dev[2]
        bm = dev[-1] if part["mask"] else None
        fa.fwd(q, k, v, causal=w.causal, scale=w.scale, out=outs[0], lse=outs[1], window=w.window,
               dropout_p=w.dropout_p, seed=w.dropout_seed, block_mask=bm)
        if w.backward:
            fa.bwd(q, k, v, outs[0], outs[1], dev[3], causal=w.causal, scale=w.scale, workspace=part["ws"],
                   dq=outs[2], dk=outs[3], dv=outs[4], window=w.window, dropout_p=w.dropout_p,
                   seed=w.dropout_seed, block_mask=bm)

    def step():
        for part in parts:
            run(part, part["dev"], part["outs"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_device_status(None) != fa.FA_OK:
        raise SystemExit("device status not clean after warm-up")

    sampler = ClockSampler(local)
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
    sampler.stop()
    barrier()
    fa.fa_kernel_timing(False)
    ms_local = e0.elapsed_time(e1)
    ms = max_over_ranks(ms_local)
    fwd_ms, nfwd = fa.fa_kernel_time_ms(0)
    bwd_ms, nbwd = fa.fa_kernel_time_ms(1)
    status = fa.fa_device_status(None)
    if status != fa.FA_OK:
        raise SystemExit(f"device status {status} after the timed region")
    clocks = sampler.summary()

    # FLOPs of one step on this rank (weak: the whole workload; strong: its share), and of
    # the whole job per step.
    share = sum(p["dev"][0].shape[0] * p["dev"][0].shape[1] for p in parts) / (w.B * w.Hq)
    step_flops_full = w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)
    job_flops = step_flops_full * (world if args.scaling == "weak" else 1)
    value = job_flops * args.steps / (ms / 1e3) / 1e12

    # ---- end to end through the public API: pinned host inputs in, results back to host
    host_in = [t.pin_memory() for p in parts for t in p["host"]]
    dev_in = [[t for p in parts for t in p["dev"]],
              [torch.empty_like(t) for p in parts for t in p["dev"]]]
    dev_out = [[t for p in parts for t in p["outs"]],
               [torch.empty_like(t) for p in parts for t in p["outs"]]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out[0]] for _ in range(2)]

    def compute(sl):
        i_in = i_out = 0
        for p in parts:
            n_in, n_out = len(p["dev"]), len(p["outs"])
            run(p, dev_in[sl][i_in:i_in + n_in], dev_out[sl][i_out:i_out + n_out])
            i_in += n_in
            i_out += n_out

    e2e_steps = max(8, args.steps // 10)
    e2e_ms = max_over_ranks(_e2e_pipelined(host_in, dev_in, dev_out, host_out, compute, e2e_steps, 2,
                                           barrier))
    nbytes = lambda *ts: sum(t.numel() * t.element_size() for t in ts)
    h2d = nbytes(*dev_in[0])
    d2h = nbytes(*dev_out[0])
    e2e_value = job_flops * e2e_steps / (e2e_ms / 1e3) / 1e12

    peaks, peak_src = _peaks()
    peak = float(peaks["bf16_tflops"])
    # Secondary bound: one exponential per visible score in each pass (the backward
    # recomputes them), at 16 per clock per SM on the MUFU unit.
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    exp_rate = 16.0 * sms * mhz * 1e6
    # The forward kernel that ran: the persistent one for dense full / causal attention
    # with d <= 128 (and its dropout form) when that scheduler is selected.
    dense = w.block_density == 0 and w.window is None
    fwd_name = ("fa_fwd_d256_kernel" if w.d == 256 else
                "fa_fwd_persist_kernel" if dense and fa.fa_get_fwd_scheduler() else "fa_fwd_kernel")
    bwd_name = _bwd_kernel_name(w)
    kernels = {}
    for kname, kms, kn, kflops in ((fwd_name, fwd_ms, nfwd, w.fwd_flops() * share / max(len(parts), 1)),
                                   (bwd_name, bwd_ms, nbwd, w.bwd_flops() * share / max(len(parts), 1))):
        if not kn:
            continue
        per = kms / kn
        exps = w.score_pairs() * share / len(parts)
        kernels[kname] = {"ms_per_launch": per, "tflops": kflops / (per / 1e3) / 1e12,
                          "tensor_bound_ms": kflops / (peak * 1e12) * 1e3,
                          "exp2_per_launch": exps,
                          "mufu_bound_ms": exps / exp_rate * 1e3,
                          "mufu_bound_note": (f"all exponentials on MUFU ex2 at 16/clk/SM x {sms} SMs x "
                                              f"{mhz:.0f} MHz (the forward runs 1/16 of them on the FMA pipe)")}
    for kname, kd in kernels.items():
        kd["frac_of_burst_peak"] = kd["tflops"] / peak
        kd["frac_of_sustained_peak"] = kd["tflops"] / float(peaks["bf16_tflops_sustained"])
        kd["frac_of_nominal_peak"] = kd["tflops"] / NOMINAL_BF16_TFLOPS
    # Dominant kernel: the backward main kernel (or the forward when there is no backward).
    dom_name = bwd_name if bwd_name in kernels else fwd_name
    achieved = kernels[dom_name]["tflops"]
    traffic = _profile_traffic(dom_name, w.name) if args.scaling == "weak" else None

    cfg = _config(w, world)
    if args.scaling == "strong":
        cfg.update(B_per_gpu=None, global_batch=w.B, parallelism=f"groups{world}",
                   groups_per_gpu=sum(p["dev"][1].shape[0] * p["dev"][1].shape[1] for p in parts))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": args.scaling, "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": cfg,
        "frac_of_peak": value / world / peak,
        "roofline": {"bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "overlap": E2E_OVERLAP},
        "gpu_launches": args.steps * len(parts) * (1 + (3 if w.backward else 0)),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        import oracle
        oracle.use_build("native")
        cores = _cores()
        oracle.set_threads(cores)
        dt, fl, groups = _oracle_groups(w, w.Hkv, w.seed, budget_s=args.cpu_budget)
        line["cpu_baseline"] = _cpu_baseline_line(w, dt, fl, groups, cores, "wall, one pass")
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
    oracle.use_build("native")
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
        oracle.use_build("native")
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_8k_causal")
    ap.add_argument("--scaling", choices=("weak", "strong"), default="weak",
                    help="weak: each rank runs the whole workload on its own batch; strong: the "
                         "workload's (batch row, K/V head) groups are split across the ranks")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle time in the CPU-baseline sample (whole K/V-head groups)")
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
