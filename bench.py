#!/usr/bin/env python
"""Benchmark of the fused attention forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 5] [--decode 1] [--backward] [--fp8]

A step is one full forward (one kernel launch) over the workload's tensors,
which are resident in device memory before the timed region starts. The
default workload is the long-context causal case (B=1, H=32, N=16384, d=128),
the largest configuration; its inputs (3 x 128 MiB) exceed the 126 MB L2 by more
than half again, so no L2 flush is done between steps. A workload whose inputs are
smaller is timed with a 256 MiB buffer written before each step, and each step
is timed alone. Metric: counted FLOPs 4*B*H*N^2*d (half when causal) per second,
in TFLOP/s.

With N > 1 GPUs (torchrun, one process per GPU) every rank runs its own
replica of the workload (own seed): there is no data exchange on the path,
only a barrier and a max-reduction of the timings ("scaling": "weak").

--impl reference times the CPU oracle (fp64 C, the machine's host cores) on a
bounded row sample of the same workload, in the same unit; under torchrun only
rank 0 runs it.

--backward times the backward pass (fa_bwd) on the workload's shape instead.
--fp8 times the e4m3 forward (fa_fwd_fp8) on the workload's shape instead.
--decode 1 times the split-KV path instead (one query row per head against an
8K-key cache with grouped K/V heads), in GB/s of algorithmic bytes; --decode 2 the
same for one sequence against a 128K-key cache (keys split into ranges and merged).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = ("attention fwd TFLOP/s (4·B·H·N²·d) and % of B200 "
          "dense BF16 peak")
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["io_aware_exact_18_b200/csrc/fa_fwd_kernel.cuh",
                  "io_aware_exact_18_b200/csrc/sm100_ptx.cuh",
                  "io_aware_exact_18_b200/csrc/fa_api.cu"]


# ----------------------------------------------------------------- helpers
L2_BYTES = 126 * 10**6          # B200 L2 cache
FLUSH_BYTES = 256 * 2**20        # written before each timed step when inputs are small


def l2_policy(input_bytes: int):
    """Whether the timed steps flush the L2, and the line that says so.

    Inputs of at least 1.5 x the 126 MB L2 stand for a cold cache by themselves
    (a step cannot find most of them still cached from the step before); smaller
    ones are timed with a 256 MiB buffer written before every step, each step
    timed alone by its own pair of events."""
    mib = input_bytes / 2**20
    if input_bytes >= 1.5 * L2_BYTES:
        return False, f"no flush: the step's inputs ({mib:.0f} MiB) exceed 1.5 x the 126 MB L2"
    return True, (f"flush: the step's inputs ({mib:.0f} MiB) are under 1.5 x the 126 MB L2, "
                  f"so a {FLUSH_BYTES >> 20} MiB buffer is written before each timed step, "
                  "which is timed alone")


def tensor_bytes(*xs) -> int:
    return sum(x.numel() * x.element_size() for x in xs)


def time_steps(torch, stream, step, steps: int, flush_buf=None) -> float:
    """Device time of one step in ms, from CUDA events on the launching stream.
    Without a flush buffer one pair of events brackets all the steps; with one,
    the buffer is overwritten before every step and each step has its own pair,
    so the flush is not timed."""
    if flush_buf is None:
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                step()
        ev1.record(stream)
        stream.synchronize()
        return ev0.elapsed_time(ev1) / steps
    pairs = []
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush_buf.fill_(i & 0xFF)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            pairs.append((a, b))
    stream.synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs) / steps


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """sha256/16 of the forward kernel's sources with comments and blank space
    removed, so that edits to comments alone keep a recorded measurement."""
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """DRAM bytes per launch from the committed ncu record, if it was taken on
    the current kernel sources: {"read": R, "write": W, "case": ...}, else
    None. Writes that are still dirty in L2 when the kernel ends are not in W
    (they reach DRAM later), so W can sit below the O + lse bytes."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload_name}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                key, val = line.split(":", 1)
                vals[key.strip()] = val.strip()
    if vals.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return {"read": float(vals["dram_read_bytes_per_launch"]),
                "write": float(vals["dram_write_bytes_per_launch"]),
                "case": vals.get("measured_case", "")}
    except (KeyError, ValueError):
        return None


def visible_pairs(w, kv_len=None) -> int:
    """Number of visible (query row, key) pairs over all B*H heads of a square
    workload: key j is visible to row i iff j < kv_len[b] (clamped to [0, N])
    and, when causal, j <= i."""
    import numpy as np
    kv_lims = [w.N] * w.B if kv_len is None else [min(max(int(x), 0), w.N) for x in kv_len]
    rows = np.arange(w.N, dtype=np.int64)
    vis = 0
    for lim in kv_lims:
        vis += int(np.minimum(lim, rows + 1).sum()) if w.causal else lim * w.N
    return vis * w.H


class ClockSampler:
    """Samples SM clock, power and clock-event (throttle) reasons in a
    background thread through NVML every 20 ms; read-only queries."""
    PERIOD_S = 0.02

    def __init__(self, torch_device_index: int):
        self.dev = torch_device_index
        self.samples = []          # (time, sm_mhz, max_mhz, power_w, reasons:set)
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._h = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        self._nvml = pynvml
        props = torch.cuda.get_device_properties(self.dev)
        try:
            bus = "{:08X}:{:02X}:{:02X}.0".format(props.pci_domain_id, props.pci_bus_id,
                                                 props.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:  # noqa: BLE001 - fall back to the visible index
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.dev]) if vis else self.dev
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            self._h = self._handle()
        except Exception:  # noqa: BLE001 - no NVML: report no samples
            self._h = None
            return
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        n = self._nvml
        names = {n.nvmlClocksEventReasonHwSlowdown: "hw_slowdown",
                 n.nvmlClocksEventReasonHwThermalSlowdown: "hw_thermal_slowdown",
                 n.nvmlClocksEventReasonSwThermalSlowdown: "sw_thermal_slowdown",
                 n.nvmlClocksEventReasonSwPowerCap: "sw_power_cap",
                 n.nvmlClocksEventReasonHwPowerBrakeSlowdown: "hw_power_brake_slowdown"}
        while not self._stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                mx = n.nvmlDeviceGetMaxClockInfo(self._h, n.NVML_CLOCK_SM)
                pw = n.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                bits = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                rs = {name for bit, name in names.items() if bits & bit}
                self.samples.append((time.time(), sm, mx, pw, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.PERIOD_S)

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, t0, t1):
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        window = "timed"
        if len(inside) < 3:
            inside = self.samples
            window = "warmup+timed"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        sm = sorted(x[1] for x in inside)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(x[2] for x in inside),
                "reasons": sorted(set().union(*[x[4] for x in inside])),
                "samples": len(inside), "window": window,
                "power_w_max": max(x[3] for x in inside), "source": "nvml, 20 ms"}


# ----------------------------------------------------------------- CPU oracle sample
def oracle_sample_rows(w, budget_s, seed, nthreads, q, k, v, kv_len, max_rows=None):
    """Time the oracle on a seeded row sample sized to about `budget_s`.

    Returns (seconds, counted_flops, description). Counted FLOPs of a row are
    4*d*(visible keys of that row); summed over all rows this is the
    metric's count."""
    import numpy as np
    import oracle
    N, d = w.N, w.d
    rng = np.random.default_rng(seed)

    def visible(i, b):
        lim = N
        if kv_len is not None:
            lim = int(min(max(int(kv_len[b]), 0), N))
        return min(lim, i + 1) if w.causal else lim

    def run(rows):
        t = time.perf_counter()
        oracle.attention(q, k, v, w.scale, causal=w.causal, kv_len=kv_len, rows=rows,
                         nthreads=nthreads)
        dt = time.perf_counter() - t
        fl = sum(4.0 * d * visible(i, b) for b in range(w.B) for i in rows) * w.H
        return dt, fl

    n_rows = 4
    while True:
        rows = sorted(set(rng.integers(0, N, size=n_rows).tolist()))
        dt, fl = run(rows)
        if dt >= 0.5 * budget_s or n_rows >= N or (max_rows and n_rows >= max_rows):
            break
        grow = 2.0 if dt <= 0 else min(8.0, max(1.5, 0.8 * budget_s / dt))
        n_rows = int(min(N, n_rows * grow))
        if max_rows:
            n_rows = min(n_rows, max_rows)
    desc = (f"{len(rows)} seeded random query rows x all {w.B * w.H} (b,h) heads of "
            f"{w.name} (fraction {len(rows) / N:.4f} of the rows), fp64, "
            f"{nthreads} threads")
    return dt, fl, desc


def reference_arm(args, w):
    """CPU oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    q, k, v, kv_len = workloads.make_inputs(w)
    nthreads = os.cpu_count() or 1
    oracle.load()
    per_step = max(0.2, min(5.0, 150.0 / max(args.steps + args.warmup, 1)))
    for i in range(args.warmup):
        oracle_sample_rows(w, per_step / 4, 10 + i, nthreads, q, k, v, kv_len)
    tot_t, tot_f, desc = 0.0, 0.0, ""
    for i in range(args.steps):
        dt, fl, desc = oracle_sample_rows(w, per_step, 1000 + i, nthreads, q, k, v, kv_len)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    # ms per step expressed for the whole workload (extrapolated from the samples)
    ms_full = w.flops() / (value * 1e12) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_full, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**w.describe(), "l2": "n/a (CPU)",
                   "note": "per-step time extrapolated from the row sample"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm
def decode_kernel_name(w, splits: int) -> str:
    """The kernels a split-KV call of decode workload w launches: the
    transposed decoding tile when the query heads of a K/V group times the
    query rows fit its 8 columns at d = 128, else the general kernel; then the
    merge when there is more than one key range."""
    tile = (w.d == 128 and (w.H // w.H_kv) * w.Nq <= 8)
    name = "fa_decode_sm100<128,bf16>" if tile else f"fa_fwd_sm100<{w.d},1,general>"
    return name + (f" + fa_splitkv_combine<{w.d}>" if splits > 1 else "")


def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() \
        and dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def square_call(fa, w, qd, kd, vd, od, lsed, kvd, sh):
    """One forward launch of a square workload through the C ABI."""
    if w.kv_heads != w.H:
        st = fa.fa_fwd_gqa(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                           lsed.data_ptr(), w.B, w.H, w.kv_heads, w.N, w.d, w.scale,
                           int(w.causal), None if kvd is None else kvd.data_ptr(), sh)
    elif kvd is None:
        st = fa.fa_fwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                       lsed.data_ptr(), w.B, w.H, w.N, w.d, w.scale, int(w.causal), sh)
    else:
        st = fa.fa_fwd_kvlen(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                             lsed.data_ptr(), w.B, w.H, w.N, w.d, w.scale, int(w.causal),
                             kvd.data_ptr(), sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "fa_fwd")


def time_workload(torch, fa, w, dev, stream, steps, warmup, seed):
    """Device time of one forward launch of workload w (ms), with its inputs
    resident in HBM and the L2 policy of l2_policy; returns (ms, l2 note)."""
    q, k, v, kv_len = workloads.make_inputs(w, seed=seed)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    kvd = None if kv_len is None else kv_len.to(dev)
    od = torch.empty_like(qd)
    lsed = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    sh = stream.cuda_stream

    def step():
        square_call(fa, w, qd, kd, vd, od, lsed, kvd, sh)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    stream.synchronize()
    step_inputs = (qd, kd, vd) if kvd is None else (qd, kd, vd, kvd)
    flush, l2_note = l2_policy(tensor_bytes(*step_inputs))
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    ms = time_steps(torch, stream, step, steps, flush_buf)
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, f"timed region of {w.name}")
    return ms, l2_note


def config_entry(w, ms, world, peak, l2_note):
    tflops = world * w.flops() / (ms * 1e-3) / 1e12
    return {"workload": w.name, "ms_per_launch": ms, "tflops": tflops,
            "frac_of_measured_peak": tflops / world / peak, "l2": l2_note}


def our_arm(args, w):
    import datetime

    import torch
    import torch.distributed as dist

    import io_aware_exact_18_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.load_library()

    # ---- inputs resident in HBM before the timed region
    q, k, v, kv_len = workloads.make_inputs(w, seed=w.index + 1000 * rank)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    kvd = None if kv_len is None else kv_len.to(dev)
    od = torch.empty_like(qd)
    lsed = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def step():
        square_call(fa, w, qd, kd, vd, od, lsed, kvd, sh)

    sampler = ClockSampler(local)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "warm-up")

    # ---- timed region: device events on the launching stream
    step_inputs = (qd, kd, vd) if kvd is None else (qd, kd, vd, kvd)
    flush, l2_note = l2_policy(tensor_bytes(*step_inputs))
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ms_local = time_steps(torch, stream, step, args.steps, flush_buf)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.stop()
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed region")
    ms = max_over_ranks(ms_local, world)
    flops = w.flops()
    value = world * flops / (ms * 1e-3) / 1e12
    clocks = sampler.summary(t_wall0, t_wall1)

    # ---- end to end through the public API with host buffers
    e2e_steps = max(1, min(args.steps, 10))
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    kvh = None if kv_len is None else kv_len.pin_memory()
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    lh = torch.empty(lsed.shape, dtype=lsed.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh)) + \
        (0 if kvh is None else kvh.numel() * kvh.element_size())
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    # Steps are pipelined the way a caller streaming batches would run them: two
    # sets of device buffers; step i's host-to-device copies (copy stream), its
    # attention call (the launching stream) and its device-to-host copies (a
    # second copy stream) are ordered by events, so step i+1's inputs cross PCIe
    # while step i computes and step i-1's result comes back. Every step still
    # copies its own inputs in and its own O and lse out inside the timed region.
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    bufs = [(qd, kd, vd, kvd, od, lsed)]
    bufs.append(tuple(None if x is None else torch.empty_like(x) for x in bufs[0]))
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_d2h:
        e.record(stream)
    e2e_count = [0]

    def e2e_step():
        b = e2e_count[0] & 1
        e2e_count[0] += 1
        q_b, k_b, v_b, kv_b, o_b, l_b = bufs[b]
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(ev_comp[b])          # the buffer's previous step has read it
            q_b.copy_(qh, non_blocking=True)
            k_b.copy_(kh, non_blocking=True)
            v_b.copy_(vh, non_blocking=True)
            if kvh is not None:
                kv_b.copy_(kvh, non_blocking=True)
            ev_h2d[b].record(h2d_stream)
        stream.wait_event(ev_h2d[b])
        stream.wait_event(ev_d2h[b])                   # its previous O and lse have left
        with torch.cuda.stream(stream):
            fa.attention(q_b, k_b, v_b, scale=w.scale, causal=w.causal, kv_len=kv_b, out=o_b,
                         lse=l_b, stream=sh)
            ev_comp[b].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev_comp[b])
            oh.copy_(o_b, non_blocking=True)
            lh.copy_(l_b, non_blocking=True)
            ev_d2h[b].record(d2h_stream)

    e2e_step()
    e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(h2d_stream)
    stream.wait_event(e0)
    d2h_stream.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    d2h_stream.wait_event(ev_d2h[0])
    d2h_stream.wait_event(ev_d2h[1])
    e1.record(d2h_stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "e2e")
    e2e_value = world * flops / (e2e_ms * 1e-3) / 1e12

    # ---- visible (query, key) pairs: the exponentials the method needs and the
    # FLOPs of the keys that are not masked (the metric counts nominal FLOPs)
    vis = visible_pairs(w, kv_len)
    eff_flops = 4.0 * w.d * vis

    # ---- roofline of the (only) kernel: one launch per step
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_local * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    rec = recorded_traffic(w.name)
    alg_read = float(w.B * w.N * (w.H + 2 * w.kv_heads) * w.d * 2)      # Q, K, V once
    alg_write = float(w.B * w.N * w.H * (w.d * 2 + 4))                   # O, lse once
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": None if rec is None else rec["read"] + rec["write"],
                "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
                "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                "frac_of_datasheet_2250": achieved / DATASHEET_BF16_TFLOPS,
                "algorithmic_bytes": alg_read + alg_write,
                "traffic_read": None if rec is None else rec["read"],
                "traffic_write": None if rec is None else rec["write"],
                "read_over_algorithmic": None if rec is None else rec["read"] / alg_read,
                "write_over_algorithmic": None if rec is None else rec["write"] / alg_write,
                "traffic_note": ("ncu dram__bytes_read.sum / dram__bytes_write.sum of one launch"
                                 + ("" if rec is None else f" ({rec['case']})")
                                 + "; reads are compared with Q + K + V, writes with O + lse; "
                                 "writes still dirty in L2 when the kernel ends are not counted"),
                # secondary bound: one exponential per visible score; MUFU ex2 runs 16 per
                # clock per SM (148 SMs) at the sampled SM clock
                "exp_per_s": vis / (ms_local * 1e-3),
                "exp_frac_of_mufu": vis / (ms_local * 1e-3) / (
                    16 * 148 * float(clocks.get("sm_mhz") or 1965) * 1e6),
                "effective_tflops_visible_keys": eff_flops / (ms_local * 1e-3) / 1e12,
                "kernel": f"fa_fwd_sm100<{w.d},{1 if w.d == 256 else 2},square>"}

    # ---- every square workload in this process, each under its own L2 policy
    # (the headline workload's entry is the measurement above)
    configs = None
    if not args.no_configs and args.shape is None:
        del qd, kd, vd, od, kvd, flush_buf
        torch.cuda.empty_cache()
        configs = []
        for cw in workloads.WORKLOADS:
            if cw.name == w.name:
                configs.append(config_entry(cw, ms, world, peak, l2_note))
                continue
            cms, cnote = time_workload(torch, fa, cw, dev, stream, args.steps, args.warmup,
                                       seed=cw.index + 1000 * rank)
            configs.append(config_entry(cw, max_over_ranks(cms, world), world, peak, cnote))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nthreads = os.cpu_count() or 1
        dt, fl, desc = oracle_sample_rows(w, args.cpu_seconds, 7, nthreads, q, k, v, kv_len)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
               "sample": desc, "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {**w.describe(), "parallelism": f"replicas x{world}",
                       "l2": l2_note},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "schedule": "pipelined: two device buffer sets; each step's host-to-device "
                                "copies, call and device-to-host copies on three streams, so "
                                "one step's copies overlap its neighbours' compute"},
            "gpu_launches": args.steps,
            "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def decode_arm(args, w):
    """Split-KV decoding: one fa_fwd_splitkv call per step (the attention
    kernel over all key ranges, then the log-sum-exp merge) at the library's
    default number of ranges. Memory-bound: reported in GB/s of algorithmic
    bytes (K, V and Q read once, O and lse written once) against the measured
    copy bandwidth. Replicas only under torchrun, like the square arm."""
    import datetime

    import torch
    import torch.distributed as dist

    import io_aware_exact_18_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.load_library()
    q, k, v, _ = workloads.make_qkv(w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d, seed=w.seed + 1000 * rank)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    od = torch.empty_like(qd)
    lsed = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    splits = fa.fa_splitkv_default_splits(w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d)
    ws_bytes = fa.fa_splitkv_workspace_bytes(w.B, w.H, w.Nq, w.d, splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def step():
        st = fa.fa_fwd_splitkv(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                               lsed.data_ptr(), w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d, w.scale,
                               int(w.causal), None, splits, ws.data_ptr(), ws_bytes, sh)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_fwd_splitkv")

    sampler = ClockSampler(local)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    step_inputs = (qd, kd, vd)
    flush, l2_note = l2_policy(tensor_bytes(*step_inputs))
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ms_local = time_steps(torch, stream, step, args.steps, flush_buf)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.stop()
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed region")
    ms = max_over_ranks(ms_local, world)
    nbytes = w.algorithmic_bytes()
    value = world * nbytes / (ms * 1e-3) / 1e9
    clocks = sampler.summary(t_wall0, t_wall1)

    # end to end: the step's inputs (q and the K/V cache) copied from pinned
    # host memory, the call, O and lse read back
    e2e_steps = max(1, min(args.steps, 5))
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    lh = torch.empty(lsed.shape, dtype=lsed.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    def e2e_step():
        with torch.cuda.stream(stream):
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            fa.decode_attention(qd, kd, vd, scale=w.scale, causal=w.causal, num_splits=splits,
                                out=od, lse=lsed, workspace=ws, stream=sh)
            oh.copy_(od, non_blocking=True)
            lh.copy_(lsed, non_blocking=True)

    e2e_step()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e_value = world * nbytes / (e2e_ms * 1e-3) / 1e9

    peaks, peak_src = load_peaks()
    achieved = nbytes / (ms_local * 1e-3) / 1e9
    peak = float(peaks["hbm_gbs"])
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": None,
                "peak_source": f"{peak_src} copy bandwidth",
                "algorithmic_bytes": float(nbytes),
                "timed": "whole step: attention kernel over all key ranges + merge kernel",
                "kernel": decode_kernel_name(w, splits)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        nthreads = os.cpu_count() or 1
        t = time.perf_counter()
        oracle.attention(q, k, v, w.scale, causal=w.causal, nthreads=nthreads)
        dt = time.perf_counter() - t
        cpu = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": nthreads, "kind": "oracle",
               "sample": f"the whole step ({w.B * w.H} query rows x {w.Nk} keys), fp64, "
                         f"{nthreads} threads", "seconds": dt}
    if rank == 0:
        line = {
            "metric": "split-KV decode attention GB/s (K, V, Q read once; O, lse written once)",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**w.describe(), "num_splits": splits,
                       "parallelism": f"replicas x{world}",
                       "l2": l2_note},
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": args.steps * (2 if splits > 1 else 1),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def backward_arm(args, w):
    """Backward pass: one fa_bwd call per step (the row-statistics kernel, the
    dK/dV pass and the dQ pass) on the workload's shape, with O and lse from
    this library's forward and dO ~ N(0,1) resident in HBM. Metric: the
    backward's algorithmic FLOPs, 2.5 x the forward's (five N x N x d products:
    S, dP, dV, dK, dQ), per second; the dQ pass recomputes S and dP, so the
    tensor cores do 7/5 of that count. Replicas only under torchrun."""
    import datetime

    import torch
    import torch.distributed as dist

    import io_aware_exact_18_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.load_library()
    H_kv = w.kv_heads
    q, k, v, do, _ = workloads.make_bwd_inputs(w.B, w.H, H_kv, w.N, w.d,
                                               seed=w.index + 100 + 1000 * rank,
                                               q_mult=w.q_mult)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o, lse = fa.attention(qd, kd, vd, scale=w.scale, causal=w.causal)
    dq, dk, dv = (torch.empty_like(x) for x in (qd, kd, vd))
    ws_bytes = fa.fa_bwd_workspace_bytes(w.B, w.H, w.N)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def step():
        st = fa.fa_bwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                       lse.data_ptr(), dod.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                       dv.data_ptr(), w.B, w.H, H_kv, w.N, w.d, w.scale, int(w.causal), None,
                       ws.data_ptr(), ws_bytes, sh)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_bwd")

    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    step_inputs = (qd, kd, vd, o, lse, dod)
    flush, l2_note = l2_policy(tensor_bytes(*step_inputs))
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ms_local = time_steps(torch, stream, step, args.steps, flush_buf)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.stop()
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed region")
    ms = max_over_ranks(ms_local, world)
    flops = 2.5 * w.flops()
    value = world * flops / (ms * 1e-3) / 1e12
    clocks = sampler.summary(t_wall0, t_wall1)

    # end to end: q, k, v, o, lse, dO copied in from pinned host memory, the
    # call, the three gradients read back
    e2e_steps = max(1, min(args.steps, 5))
    hin = [x.pin_memory() for x in (q, k, v, o.cpu(), lse.cpu(), do)]
    dins = [qd, kd, vd, o, lse, dod]
    hout = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in (dq, dk, dv)]
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = sum(x.numel() * x.element_size() for x in hout)

    def e2e_step():
        with torch.cuda.stream(stream):
            for dd_, hh in zip(dins, hin):
                dd_.copy_(hh, non_blocking=True)
            fa.attention_bwd(qd, kd, vd, o, lse, dod, scale=w.scale, causal=w.causal, dq=dq,
                             dk=dk, dv=dv, workspace=ws, stream=sh)
            for hh, dd_ in zip(hout, (dq, dk, dv)):
                hh.copy_(dd_, non_blocking=True)

    e2e_step()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e_value = world * flops / (e2e_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    achieved = flops / (ms_local * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None,
                "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
                "tensor_work_frac": achieved * 7 / 5 / peak,
                "timed": "whole step: row statistics + dK/dV pass + dQ pass",
                "kernel": f"fa_bwd_prep<{w.d}> + fa_bwd_dkdv<{w.d}> + fa_bwd_dq<{w.d}>"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        nthreads = os.cpu_count() or 1
        Hs, Ns = min(w.H, 16), min(w.N, 2048)
        qs, ks, vs, dos, _ = workloads.make_bwd_inputs(1, Hs, Hs, Ns, w.d, seed=3)
        t = time.perf_counter()
        oracle.attention_bwd(qs, ks, vs, dos, w.scale, causal=w.causal, nthreads=nthreads)
        dt = time.perf_counter() - t
        sflops = 10.0 * Hs * Ns * Ns * w.d * (0.5 if w.causal else 1.0)
        cpu = {"value": sflops / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
               "sample": f"the same computation at B=1, H={Hs}, N={Ns}, d={w.d} "
                         f"({'causal' if w.causal else 'full'}), fp64, {nthreads} threads",
               "seconds": dt}
    if rank == 0:
        line = {
            "metric": "attention bwd TFLOP/s (2.5 x forward FLOPs: 10·B·H·N²·d, half causal)",
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**w.describe(), "pass": "backward", "parallelism": f"replicas x{world}",
                       "l2": l2_note},
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": 3 * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def fp8_arm(args, w):
    """The e4m3 forward (fa_fwd_fp8) on the workload's shape: Q, K, V quantized
    per tensor to e4m3 (descale amax / 448) and resident in HBM, one launch per
    step. Same metric as the bf16 line (4*B*H*N^2*d, half causal); the roofline
    peak is the measured bf16 figure times the nominal e4m3 / bf16 ratio (2)."""
    import datetime

    import torch
    import torch.distributed as dist

    import io_aware_exact_18_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.load_library()
    q8, k8, v8, sc, _ = workloads.make_fp8_inputs(w.B, w.H, w.kv_heads, w.N, w.d,
                                                  seed=w.index + 200 + 1000 * rank)
    qd, kd, vd = (x.to(dev) for x in (q8, k8, v8))
    od = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    lsed = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def step():
        st = fa.fa_fwd_fp8(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), sc[0], sc[1], sc[2],
                           od.data_ptr(), lsed.data_ptr(), w.B, w.H, w.kv_heads, w.N, w.d,
                           w.scale, int(w.causal), None, sh)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_fwd_fp8")

    sampler = ClockSampler(local)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    step_inputs = (qd, kd, vd)
    flush, l2_note = l2_policy(tensor_bytes(*step_inputs))
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ms_local = time_steps(torch, stream, step, args.steps, flush_buf)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.stop()
    st = fa.fa_last_device_error(sh)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed region")
    ms = max_over_ranks(ms_local, world)
    flops = w.flops()
    value = world * flops / (ms * 1e-3) / 1e12
    clocks = sampler.summary(t_wall0, t_wall1)

    e2e_steps = max(1, min(args.steps, 10))
    hin = [x.view(torch.uint8).pin_memory() for x in (q8, k8, v8)]
    din = [x.view(torch.uint8) for x in (qd, kd, vd)]
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    lh = torch.empty(lsed.shape, dtype=lsed.dtype).pin_memory()
    h2d = sum(x.numel() for x in hin)
    d2h = oh.numel() * 2 + lh.numel() * 4

    def e2e_step():
        with torch.cuda.stream(stream):
            for dd_, hh in zip(din, hin):
                dd_.copy_(hh, non_blocking=True)
            fa.attention_fp8(qd, kd, vd, *sc, scale=w.scale, causal=w.causal, out=od, lse=lsed,
                             stream=sh)
            oh.copy_(od, non_blocking=True)
            lh.copy_(lsed, non_blocking=True)

    e2e_step()
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e_value = world * flops / (e2e_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    achieved = flops / (ms_local * 1e-3) / 1e12
    peak = 2.0 * float(peaks["bf16_tflops"])
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None,
                "peak_source": f"{peak_src} bf16 burst (cuBLAS) x nominal e4m3/bf16 ratio 2",
                "kernel": f"fa_fwd_sm100<{w.d},2,square,e4m3>"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import fp8 as ofp8
        nthreads = os.cpu_count() or 1
        rows = workloads.sample_rows(w.N, seed=9, n_random=24, edge=4)
        t = time.perf_counter()
        ofp8.attention_fp8(q8, k8, v8, *sc, w.scale, causal=w.causal, rows=rows,
                           nthreads=nthreads)
        dt = time.perf_counter() - t
        fl = sum(4.0 * w.d * ((i + 1) if w.causal else w.N) for i in rows) * w.B * w.H
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
               "sample": f"{len(rows)} query rows x all {w.B * w.H} heads of the same e4m3 "
                         f"inputs, dequantized, fp64, {nthreads} threads", "seconds": dt}
    if rank == 0:
        line = {
            "metric": METRIC + " (e4m3 inputs)", "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3", "data": "synthetic",
            "config": {**w.describe(), "inputs": "e4m3, per-tensor descale amax/448",
                       "parallelism": f"replicas x{world}",
                       "l2": l2_note},
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="5", help="workload index (1-5) or name")
    ap.add_argument("--shape", default=None,
                    help="custom B,H,N,d[,causal[,H_kv]] (smaller or grouped-query cases; "
                         "same recipe)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload timings of the five square workloads")
    ap.add_argument("--fp8", action="store_true",
                    help="time the e4m3 forward (fa_fwd_fp8) on the workload instead")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (fa_bwd) on the workload instead")
    ap.add_argument("--decode", default=None,
                    help="time the split-KV decode path on this decode workload "
                         "(name, or 1 for the first) instead of square attention")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # timing rule: at least 3 untimed warm-up steps
    if args.decode:
        dw = (workloads.DECODE_WORKLOADS[int(args.decode) - 1] if args.decode.isdigit()
              else workloads.DECODE_BY_NAME[args.decode])
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the decode line has no reference arm; its cpu_baseline key "
                              "times the oracle"}), flush=True)
            return 0
        return decode_arm(args, dw)
    if args.shape:
        f = [int(x) for x in args.shape.split(",")]
        B, H, N, d = f[:4]
        causal = bool(f[4]) if len(f) > 4 else False
        H_kv = f[5] if len(f) > 5 else None
        tag = "" if H_kv is None else f"_Hkv{H_kv}"
        w = workloads.Workload(f"custom_B{B}_H{H}{tag}_N{N}_d{d}_{'causal' if causal else 'full'}",
                               0, B, H, N, d, causal, H_kv=H_kv)
    else:
        w = workloads.get(args.workload)
    if args.fp8:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the e4m3 line has no reference arm; its cpu_baseline key "
                              "times the oracle"}), flush=True)
            return 0
        return fp8_arm(args, w)
    if args.backward:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the backward line has no reference arm; its cpu_baseline key "
                              "times the oracle"}), flush=True)
            return 0
        return backward_arm(args, w)
    if args.impl == "reference":
        return reference_arm(args, w)
    return our_arm(args, w)


if __name__ == "__main__":
    sys.exit(main())
