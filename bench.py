"""Benchmark of the grouped block-scaled quantization path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1..5]

One step (the default, config 5) is the Qwen3-235B-A22B expert
prequantization sweep: 94 layers, each layer's 128 gate_up [3072, 4096] and
128 down [4096, 1536] bf16 experts (N(0, 0.02), 4.83 GB) regenerated in place
from seed 5 + layer before the layer is timed, then quantized per projection
in one call each to
  - MXFP8 (E8M0 scales, swizzled 128x4),
  - NVFP4 with the per-tensor FP32 scale computed by the call (one
    cooperative launch: bulk copies feed the amax side, the quantize side
    re-reads from L2), and
  - NVFP4 again with that amax given (a requantization with a known scale),
six calls per layer, every call bracketed by CUDA events on the stream it
runs on.  Inputs are far larger than L2 (3.2 GB per call).  The metric is
(input + output bytes) / time in GB/s; the step time is the sum of the event
times of its 564 calls (the regeneration between layers is not timed).

The JSON line carries the roofline of every kernel of the step (algorithmic
bytes per launch over its event time, against the measured HBM copy
bandwidth; the dominant one as ``roofline``), an end-to-end figure through
the same C ABI with every layer's weights coming from pinned host memory and
the quantized bytes going back, the CPU oracle timed on a bounded sample on
one host thread and on all of them, SM clocks sampled during the timed
region, the Qwen3-30B-A3B MXFP8 refit step (config 2) as ``refit_30b``, and
(``extra``) the other workloads: the tiny MXFP8 group, the row-scaled NVFP4
split activation, the fused residual + RMSNorm + quantize sweep and its
AllReduce form over 8 rank buffers, the Qwen3-30B-A3B gate_up layer in NVFP4,
dequantization, column-wise quantization, the attention decode merge and the
gate|up split.

With torchrun (N > 1) every rank quantizes its own full workload on its own
GPU (weak scaling, no collective on the data path); the time is the maximum
over ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "grouped MXFP8/NVFP4 quantize GB/s (in+out bytes), % of B200 HBM peak"
FALLBACK_HBM_GBS = 6650.0
GB = 1e9


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The source files each timed kernel is built from (its own file plus the
# shared device helpers): a traffic figure stays valid while these are unchanged.
KERNEL_SOURCES = {
    "mxfp8_grouped_kernel": ("qz_grouped.cu", "qz_device.cuh"),
    "nvfp4_tile_kernel": ("qz_grouped.cu", "qz_device.cuh"),
    "nvfp4_compute_pipe_kernel": ("qz_grouped.cu", "qz_device.cuh"),
    "nvfp4_rows_kernel": ("qz_rows.cu", "qz_device.cuh"),
    "rmsnorm_quant_kernel": ("qz_rmsnorm.cu", "qz_device.cuh"),
    "rmsnorm_quant_kernel_multi": ("qz_rmsnorm.cu", "qz_device.cuh"),   # the AllReduce instantiation
    "dequant_kernel": ("qz_dequant.cu", "qz_device.cuh"),
    "attention_merge_kernel": ("qz_merge.cu", "qz_device.cuh"),
    "colwise_kernel": ("qz_colwise.cu", "qz_device.cuh", "qz_async.cuh"),
    "split_fused_kernel": ("qz_split.cu", "qz_device.cuh"),
}


def kernel_sources_sha(kernel: str) -> str:
    """sha256 (first 16 hex digits) over the named kernel's source files."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_quantization_moe_b200", "csrc")
    for f in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str = ""):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or
    None when the summary was taken on other kernel sources (or, with
    `workload`, for a workload whose tag does not start with it)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    if not os.path.exists(path):
        return None
    sha = kernel_sources_sha(kernel)
    pat = re.compile(r"^traffic: kernel=(\S+) workload=(\S+) bytes_per_launch=(\d+) sources_sha=(\w+)")
    with open(path) as f:
        for line in f:
            m = pat.match(line.strip())
            if m and m.group(1) == kernel and m.group(4) == sha and m.group(2).startswith(workload):
                return int(m.group(3))
    return None


class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            ident = str(device_index)
        self.cmd = ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "200"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# multi-rank host logic (weak scaling, no collective on the data path)
# ---------------------------------------------------------------------------

def rank_seed_offset(rank: int) -> int:
    """Each rank quantizes its own synthetic workload: the seeds shift by rank."""
    return int(rank)


def max_over_ranks(values, device):
    """Element-wise maximum over all ranks (the slowest rank sets the time)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate_gbs(bytes_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: the bytes of all ranks over the max-over-ranks time."""
    return world * bytes_per_rank * steps / (total_ms / 1e3) / GB


# ---------------------------------------------------------------------------
# workloads (the product path: every launch goes through the C ABI)
# ---------------------------------------------------------------------------

class Refit30B:
    """Qwen3-30B-A3B MXFP8 refit prequantization, all layers resident."""

    kernel = "mxfp8_grouped_kernel"

    def __init__(self, qz, device, layers=48, per_call=16, seed_offset=0):
        cfg = synth.QWEN3_30B
        self.qz = qz
        self.layers = layers
        self.calls = []        # (table, algorithmic bytes)
        self.bytes_in = 0
        self.bytes_out = 0
        self._keep = []
        for layer in range(layers):
            for proj, shape in (("gate_up", cfg["gate_up"]), ("down", cfg["down"])):
                seed = cfg["seed"] + layer + rank_seed_offset(seed_offset) * 1000 + (0 if proj == "gate_up" else 500)
                stack = synth.expert_stack(cfg["experts"], shape, cfg["std"], seed=seed, device=device)
                rows, cols = shape
                nsf = qz.sf_bytes(rows, cols, qz.FMT_MXFP8, qz.SF_SWIZZLED)
                q = torch.empty((cfg["experts"], rows, cols), dtype=torch.uint8, device=device)
                sf = torch.empty((cfg["experts"], nsf), dtype=torch.uint8, device=device)
                self._keep.append((stack, q, sf))
                for s in range(0, cfg["experts"], per_call):
                    entries = [qz.Entry(stack[e], q[e], sf[e]) for e in range(s, s + per_call)]
                    bin_ = per_call * rows * cols * 2
                    bout = per_call * (rows * cols + nsf)
                    self.calls.append((qz.ExpertTable(entries), bin_ + bout))
                    self.bytes_in += bin_
                    self.bytes_out += bout
        self.bytes = self.bytes_in + self.bytes_out

    @property
    def launches(self):
        return len(self.calls)

    def step(self, stream, events=None, side=None, independent=False):
        """One pass over all calls.  With `side` streams, calls go round-robin
        to them (independent calls may overlap) and `stream` joins them at the
        end; per-launch events are only taken on a single stream.  With
        `independent` every call is declared independent (QZ_OPT_INDEPENDENT):
        on one stream, each call's tiles may start on the SMs the previous
        call's tail frees."""
        qz = self.qz
        if side:
            start = torch.cuda.Event()
            start.record(stream)
            for s in side:
                s.wait_event(start)
            for i, (table, _) in enumerate(self.calls):
                st = side[i % len(side)]
                if events is not None:
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(st)
                    qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=st)
                    b.record(st)
                    events.append((a, b))
                else:
                    qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=st)
            for s in side:
                done = torch.cuda.Event()
                done.record(s)
                stream.wait_event(done)
            return
        for table, _ in self.calls:
            if events is not None:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=stream)
                b.record(stream)
                events.append((a, b))
            else:
                qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=stream, independent=independent)


def time_steps(work, steps, warmup, stream, dist_ok, side=None, per_launch=True, independent=False):
    """W untimed steps, then K timed steps bracketed by barrier + sync.  With
    per_launch, CUDA events bracket every launch on its own stream (timing
    events between the launches of two streams cost their overlap, so the
    headline pass goes without them).  Returns the total ms, every launch's
    duration and the union of the launch intervals (overlaps counted once)."""
    for _ in range(warmup):
        work.step(stream, side=side, independent=independent)
    torch.cuda.synchronize()
    if dist_ok:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    launch_events = []
    start.record(stream)
    for _ in range(steps):
        work.step(stream, launch_events if per_launch else None, side=side, independent=independent)
    end.record(stream)
    torch.cuda.synchronize()
    if dist_ok:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    launch_ms = [a.elapsed_time(b) for a, b in launch_events]
    spans = sorted((start.elapsed_time(a), start.elapsed_time(b)) for a, b in launch_events)
    busy, cur_a, cur_b = 0.0, None, None
    for a, b in spans:
        if cur_b is None or a > cur_b:
            if cur_b is not None:
                busy += cur_b - cur_a
            cur_a, cur_b = a, b
        else:
            cur_b = max(cur_b, b)
    if cur_b is not None:
        busy += cur_b - cur_a
    return total_ms, launch_ms, busy


def e2e_refit(qz, device, steps, warmup, layers=48, per_call=16, pool=2):
    """The same refit step through the C ABI with host-resident weights:
    every layer's bf16 experts go host -> device (pinned), are quantized, and
    the payload + scales come back device -> host.  Copies and kernels are
    pipelined over three streams with double-buffered device staging."""
    cfg = synth.QWEN3_30B
    E = cfg["experts"]
    shapes = (cfg["gate_up"], cfg["down"])
    host_in = []
    for p in range(pool):
        host_in.append([synth.expert_stack(E, s, cfg["std"], seed=cfg["seed"] + 7000 + p * 10 + i).pin_memory()
                        for i, s in enumerate(shapes)])
    nsf = [qz.sf_bytes(r, c, qz.FMT_MXFP8, qz.SF_SWIZZLED) for r, c in shapes]
    host_q = [torch.empty((E, r, c), dtype=torch.uint8).pin_memory() for r, c in shapes]
    host_sf = [torch.empty((E, n), dtype=torch.uint8).pin_memory() for n in nsf]
    bufs = []
    for _ in range(2):
        xin = [torch.empty((E, r, c), dtype=torch.bfloat16, device=device) for r, c in shapes]
        q = [torch.empty((E, r, c), dtype=torch.uint8, device=device) for r, c in shapes]
        sf = [torch.empty((E, n), dtype=torch.uint8, device=device) for n in nsf]
        tables = []
        for i in range(2):
            for s in range(0, E, per_call):
                tables.append(qz.ExpertTable([qz.Entry(xin[i][e], q[i][e], sf[i][e]) for e in range(s, s + per_call)]))
        bufs.append((xin, q, sf, tables))
    h2d, comp, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    bytes_in = sum(E * r * c * 2 for r, c in shapes)
    bytes_out = sum(E * (r * c + n) for (r, c), n in zip(shapes, nsf))

    done_d2h = [None, None]   # last D2H out of each staging buffer, across steps

    def one_step():
        for layer in range(layers):
            b = layer & 1
            xin, q, sf, tables = bufs[b]
            src = host_in[layer % pool]
            with torch.cuda.stream(h2d):
                if done_d2h[b] is not None:
                    h2d.wait_event(done_d2h[b])
                for i in range(2):
                    xin[i].copy_(src[i], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(h2d)
            comp.wait_event(ev_in)
            for t in tables:
                qz.quantize_grouped_mxfp8(t, qz.SF_SWIZZLED, stream=comp)
            ev_c = torch.cuda.Event()
            ev_c.record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_c)
                for i in range(2):
                    host_q[i].copy_(q[i], non_blocking=True)
                    host_sf[i].copy_(sf[i], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(d2h)
                done_d2h[b] = ev_o
    for _ in range(warmup):
        one_step()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(h2d)
    for _ in range(steps):
        one_step()
    torch.cuda.current_stream().wait_stream(d2h)
    torch.cuda.current_stream().wait_stream(comp)
    torch.cuda.current_stream().wait_stream(h2d)
    end.record(torch.cuda.current_stream())
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    wall = time.perf_counter() - t0
    per_step = layers * (bytes_in + bytes_out)
    return {"value": round(steps * per_step / (ms / 1e3) / GB, 2), "unit": "GB/s",
            "h2d_bytes_per_step": layers * bytes_in, "d2h_bytes_per_step": layers * bytes_out,
            "ms_per_step": round(ms / steps, 3), "wall_s": round(wall, 3),
            "note": f"host weights from {pool} pinned layer buffers cycled over {layers} layers; "
                    "H2D, kernels and D2H pipelined on three streams"}


# ---------------------------------------------------------------------------
# the headline: Qwen3-235B-A22B prequantization sweep, every layer regenerated
# ---------------------------------------------------------------------------

PROJS = ("gate_up", "down")
SWEEP_MODES = ("mxfp8", "nvfp4_compute", "nvfp4_given")
SWEEP_KERNELS = {"mxfp8": "mxfp8_grouped_kernel", "nvfp4_compute": "nvfp4_compute_pipe_kernel",
                 "nvfp4_given": "nvfp4_tile_kernel"}


class Prequant235B:
    """Per layer: regenerate the layer's experts in place (untimed), then six
    calls -- MXFP8, NVFP4 with the per-tensor amax computed, NVFP4 with that
    amax given -- for gate_up and for down, 128 experts per call."""

    def __init__(self, qz, device, layers=94, rank=0, compute_workspace=True):
        cfg = synth.QWEN3_235B
        self.qz, self.cfg, self.layers, self.rank = qz, cfg, layers, rank
        E = cfg["experts"]
        self.x, self.calls, self.keep = {}, [], []
        self.ws = qz.alloc_workspace(E, device) if compute_workspace else None
        self.compute_launches = 1 if compute_workspace else 3
        self.kernels = dict(SWEEP_KERNELS)
        if not compute_workspace:
            self.kernels["nvfp4_compute"] = "amax_grouped_kernel+nvfp4_tile_kernel"
        self.host_out = {}   # for e2e: what a layer's outputs are (device tensors)
        for proj in PROJS:
            rows, cols = cfg[proj]
            x = torch.empty((E, rows, cols), dtype=torch.bfloat16, device=device)
            self.x[proj] = x
            nmx = qz.sf_bytes(rows, cols, qz.FMT_MXFP8, qz.SF_SWIZZLED)
            nnv = qz.sf_bytes(rows, cols, qz.FMT_NVFP4, qz.SF_SWIZZLED)
            mq = torch.empty((E, rows, cols), dtype=torch.uint8, device=device)
            msf = torch.empty((E, nmx), dtype=torch.uint8, device=device)
            nq = torch.empty((E, rows, cols // 2), dtype=torch.uint8, device=device)
            nsf = torch.empty((E, nnv), dtype=torch.uint8, device=device)
            amax = torch.zeros((E, 1), dtype=torch.float32, device=device)
            self.keep.append((mq, msf, nq, nsf, amax))
            self.host_out[proj] = (mq, msf, nq, nsf, amax)
            mtab = qz.ExpertTable([qz.Entry(x[e], mq[e], msf[e]) for e in range(E)])
            ntab = qz.ExpertTable([qz.Entry(x[e], nq[e], nsf[e], amax[e]) for e in range(E)])
            bin_ = E * rows * cols * 2
            self.calls.append(("mxfp8", proj, mtab, bin_ + E * (rows * cols + nmx)))
            self.calls.append(("nvfp4_compute", proj, ntab, bin_ + E * (rows * cols // 2 + nnv + 4)))
            self.calls.append(("nvfp4_given", proj, ntab, bin_ + E * (rows * cols // 2 + nnv + 4)))
        order = {m: i for i, m in enumerate(SWEEP_MODES)}
        self.calls.sort(key=lambda c: (order[c[0]], PROJS.index(c[1])))
        self.bytes_per_layer = sum(c[3] for c in self.calls)
        self.bytes = self.bytes_per_layer * layers
        self.launches_per_layer = sum(self.compute_launches if c[0] == "nvfp4_compute" else 1 for c in self.calls)

    def regenerate(self, layer):
        for proj in PROJS:
            synth.moe_layer(self.cfg, layer, proj, rank=self.rank, out=self.x[proj])

    def call(self, mode, table, stream):
        qz = self.qz
        if mode == "mxfp8":
            qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=stream)
        elif mode == "nvfp4_compute":
            qz.quantize_grouped_nvfp4(table, qz.NVFP4_PER_TENSOR_COMPUTE, qz.SF_SWIZZLED, stream=stream,
                                      workspace=self.ws)
        else:
            qz.quantize_grouped_nvfp4(table, qz.NVFP4_PER_TENSOR_GIVEN, qz.SF_SWIZZLED, stream=stream)

    def layer_calls(self, stream, events=None):
        for mode, proj, table, nbytes in self.calls:
            if events is not None:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                self.call(mode, table, stream)
                b.record(stream)
                events.append((mode, proj, nbytes, a, b))
            else:
                self.call(mode, table, stream)

    def step(self, stream, events=None):
        for layer in range(self.layers):
            with torch.cuda.stream(stream):
                self.regenerate(layer)
            self.layer_calls(stream, events)


def time_sweep(work, steps, warmup, stream, dist_ok):
    """W untimed steps, then K steps bracketed by barrier + synchronize; every
    call of the K steps is bracketed by CUDA events on its stream.  Returns the
    per-mode totals (ms, bytes, calls), the summed call time and the device
    time of the whole sweep including the untimed regeneration."""
    for _ in range(warmup):
        work.step(stream)
    torch.cuda.synchronize()
    if dist_ok:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    events = []
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(steps):
        work.step(stream, events)
    s1.record(stream)
    torch.cuda.synchronize()
    if dist_ok:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    per = {m: {"ms": 0.0, "bytes": 0, "calls": 0, "by_proj": {p: [0.0, 0, 0] for p in PROJS}} for m in SWEEP_MODES}
    for mode, proj, nbytes, a, b in events:
        ms = a.elapsed_time(b)
        d = per[mode]
        d["ms"] += ms
        d["bytes"] += nbytes
        d["calls"] += 1
        bp = d["by_proj"][proj]
        bp[0] += ms
        bp[1] += nbytes
        bp[2] += 1
    total_ms = sum(d["ms"] for d in per.values())
    return per, total_ms, s0.elapsed_time(s1)


def sweep_roofline(per, peak, peak_kind, launches, kernels):
    """Roofline of every kernel of the sweep: algorithmic bytes per launch over
    the launch's CUDA-event time (a call is one launch of the kernel, plus a
    workspace memset for the computed-amax call)."""
    out = {}
    for mode, d in per.items():
        achieved = d["bytes"] / (d["ms"] / 1e3) / GB
        k = kernels[mode]
        out[mode] = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic(k, "qwen3-235b-sweep") if k in KERNEL_SOURCES else None,
                     "kernel": k,
                     "launches_per_call": launches.get(mode, 1),
                     "bytes_per_launch": int(d["bytes"] / max(1, d["calls"])),
                     "mean_launch_us": round(1e3 * d["ms"] / max(1, d["calls"]), 1),
                     "by_proj": {p: {"GB/s": round(v[1] / (v[0] / 1e3) / GB, 1),
                                     "frac": round(v[1] / (v[0] / 1e3) / GB / peak, 4),
                                     "us": round(1e3 * v[0] / max(1, v[2]), 1)}
                                 for p, v in d["by_proj"].items() if v[2]}}
    dom = max(per, key=lambda m: per[m]["ms"])
    roof = dict(out[dom])
    roof["peak_source"] = "measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6650 GB/s"
    roof["timing"] = "CUDA events around every call on its stream, summed over the timed steps"
    roof["dominant"] = dom
    roof["by_mode"] = out
    return roof


def e2e_prequant(qz, device, steps, warmup, layers=4, pool=2, compute_workspace=True):
    """The sweep end to end through the C ABI: every layer's bf16 experts come
    host -> device from pinned memory, the six calls run, and every quantized
    byte (both MXFP8 and NVFP4 payloads, scales and amax) goes device -> host.
    Copies and calls are pipelined over three streams with double-buffered
    device layers."""
    cfg = synth.QWEN3_235B
    E = cfg["experts"]
    host_in = [{p: synth.moe_layer(cfg, 7000 + i, p, device=device).cpu().pin_memory() for p in PROJS}
               for i in range(pool)]
    works = [Prequant235B(qz, device, layers=1, compute_workspace=compute_workspace) for _ in range(2)]
    host_out = {p: [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in works[0].host_out[p]] for p in PROJS}
    h2d, comp, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    done_d2h = [None, None]
    h2d_bytes = sum(E * r * c * 2 for r, c in (cfg[p] for p in PROJS))
    d2h_bytes = sum(t.numel() * t.element_size() for p in PROJS for t in works[0].host_out[p])

    def one_step():
        for layer in range(layers):
            b = layer & 1
            w = works[b]
            src = host_in[layer % pool]
            with torch.cuda.stream(h2d):
                if done_d2h[b] is not None:
                    h2d.wait_event(done_d2h[b])
                for p in PROJS:
                    w.x[p].copy_(src[p], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(h2d)
            comp.wait_event(ev_in)
            w.layer_calls(comp)
            ev_c = torch.cuda.Event()
            ev_c.record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_c)
                for p in PROJS:
                    for hd, dv in zip(host_out[p], w.host_out[p]):
                        hd.copy_(dv, non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(d2h)
                done_d2h[b] = ev_o

    for _ in range(warmup):
        one_step()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    start.record(h2d)
    for _ in range(steps):
        one_step()
    cur = torch.cuda.current_stream()
    for st in (d2h, comp, h2d):
        cur.wait_stream(st)
    end.record(cur)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    wall = time.perf_counter() - t0
    per_step = layers * works[0].bytes_per_layer
    res = {"value": round(steps * per_step / (ms / 1e3) / GB, 2), "unit": "GB/s",
           "h2d_bytes_per_step": layers * h2d_bytes, "d2h_bytes_per_step": layers * d2h_bytes,
           "ms_per_step": round(ms / steps, 3), "wall_s": round(wall, 3), "layers_per_step": layers,
           "note": f"weights of {pool} pinned host layers cycled over {layers} layers per step; H2D, the six "
                   "calls and D2H of all outputs pipelined on three streams"}
    del works, host_in, host_out
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# extra workloads (one timed line each, not the headline)
# ---------------------------------------------------------------------------

def _time_graph(fn, reps=20, flush=None):
    """Median-free device time of one call: `reps` calls (each after an L2
    flush when given) captured in one CUDA graph, replayed and timed with CUDA
    events; the flush time, measured the same way, is subtracted."""
    def capture(body):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            body()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s):
                for _ in range(reps):
                    body()
        torch.cuda.current_stream().wait_stream(s)
        return g

    def run(g):
        g.replay()
        torch.cuda.synchronize()
        best = None
        for _ in range(3):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            t = a.elapsed_time(b) / reps
            best = t if best is None else min(best, t)
        return best

    if flush is None:
        return run(capture(fn))
    both = run(capture(lambda: (flush(), fn())))
    only = run(capture(flush))
    return max(both - only, 1e-6)


class L2Flush:
    def __init__(self, device):
        self.buf = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.zero_()


def extra_workloads(qz, device, stream, peak,
                    which=("tiny", "split", "fused", "nvfp4", "large", "dequant", "merge", "colwise", "gateup",
                           "allreduce"),
                    tokens=None, experts=None):
    out = []
    flush = L2Flush(device)

    def rec(name, nbytes, ms, launches, **kw):
        gbs = nbytes / (ms / 1e3) / GB
        d = {"workload": name, "GB/s": round(gbs, 1), "frac_of_hbm_peak": round(gbs / peak, 4),
             "us_per_call": round(ms * 1e3, 2), "bytes_per_call": int(nbytes), "launches_per_call": launches}
        d.update(kw)
        out.append(d)

    if "tiny" in which:
        _extra_tiny(qz, device, rec)
    if "split" in which:
        _extra_split(qz, device, flush, rec)
    if "fused" in which:
        _extra_fused(qz, device, flush, out, peak, tokens)
    if "nvfp4" in which:
        _extra_nvfp4_30b(qz, device, rec)
    if "large" in which:
        _extra_large(qz, device, rec, experts)
    if "dequant" in which:
        _extra_dequant(qz, device, rec)
    if "merge" in which:
        _extra_merge(qz, device, flush, out, peak, tokens)
    if "colwise" in which:
        _extra_colwise(qz, device, rec)
    if "gateup" in which:
        _extra_gate_up_split(qz, device, rec)
    if "allreduce" in which:
        _extra_allreduce(qz, device, out, peak, tokens)
    return out


def _extra_tiny(qz, device, rec):
    """The tiny MXFP8 group (4 experts [64, 256], linear scales): a
    launch-latency case.  Reports the median and the 10th / 90th percentile of
    200 single calls, each bracketed by CUDA events; all of them are queued
    behind a spinning kernel first, so the events see the device time of each
    call and not the host's launch overhead."""
    xs = [x.to(device) for x in synth.tiny_group()]
    ents = qz.alloc_outputs(xs, qz.FMT_MXFP8, qz.SF_LINEAR, qz.NVFP4_PER_ROW)
    tab = qz.ExpertTable(ents)
    for _ in range(20):
        qz.quantize_grouped_mxfp8(tab, qz.SF_LINEAR)
    torch.cuda.synchronize()
    n = 200
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda._sleep(40_000_000)  # ~20 ms of device time: the host queues every call meanwhile
    for a, b in ev:
        a.record()
        qz.quantize_grouped_mxfp8(tab, qz.SF_LINEAR)
        b.record()
    torch.cuda.synchronize()
    times = sorted(a.elapsed_time(b) for a, b in ev)
    ms = _time_graph(lambda: qz.quantize_grouped_mxfp8(tab, qz.SF_LINEAR), reps=50)
    rows, cols = xs[0].shape
    nbytes = len(xs) * (rows * cols * 3 + rows * cols // 32)
    rec("tiny MXFP8 group: 4 experts [64, 256], linear scales", nbytes, ms, 1, kernel="mxfp8_grouped_kernel",
        timing="per call of a CUDA graph of 50 calls; single_call_* from 200 calls each bracketed by CUDA events "
               "(event pair included), all queued behind a spinning kernel",
        single_call_median_us=round(times[len(times) // 2] * 1e3, 2),
        single_call_p10_us=round(times[len(times) // 10] * 1e3, 2),
        single_call_p90_us=round(times[9 * len(times) // 10] * 1e3, 2))


def _extra_split(qz, device, flush, rec):
    """Row-scaled NVFP4 split activation [16384, 4096] over 64 experts.  Two
    copies of the input and of every output are quantized alternately, so
    consecutive calls share no bytes (2 x 173 MB moved, more than L2 holds)
    and no flush buffer leaves dirty lines for the timed calls to write back."""
    x0 = synth.split_activation(device=device)
    counts = synth.dirichlet_splits()
    T, K = x0.shape
    tables, nsf_tot = [], 0
    for copy in range(2):
        x = x0 if copy == 0 else x0.clone()
        q = torch.empty((T, K // 2), dtype=torch.uint8, device=device)
        am = torch.empty(T, dtype=torch.float32, device=device)
        entries, off, nsf_tot = [], 0, 0
        for c in counts:
            c = int(c)
            n = qz.sf_bytes(c, K, qz.FMT_NVFP4, qz.SF_SWIZZLED)
            sf = torch.empty(max(n, 16), dtype=torch.uint8, device=device)
            entries.append(qz.Entry(x[off:off + c], q[off:off + c], sf, am[off:off + c]))
            nsf_tot += n
            off += c
        tables.append(qz.ExpertTable(entries))
    turn = [0]

    def split_call():
        qz.quantize_grouped_nvfp4(tables[turn[0] % 2], qz.NVFP4_PER_ROW, qz.SF_SWIZZLED)
        turn[0] += 1

    ms = _time_graph(split_call, reps=10)
    nbytes = T * K * 2 + T * K // 2 + nsf_tot + T * 4
    rec("row-scaled NVFP4 split [16384,4096] over 64 Dirichlet(0.3) experts, swizzled", nbytes, ms, 1,
        kernel="nvfp4_rows_kernel",
        l2="inputs larger than L2: two copies of input and outputs alternated (no flush)",
        timing="CUDA graph of 10 calls", traffic=ncu_traffic("nvfp4_rows_kernel"))
    del x0, tables


def _extra_fused(qz, device, flush, out, peak, tokens=None):
    """Fused residual + RMSNorm + quantize, T sweep at H = 7168.  From
    T = 1024 on, enough copies of inputs and outputs are used round-robin that
    a call's bytes were last touched more than twice the L2 size ago (no
    flush, so no dirty flush lines are written back inside the timed calls);
    below, calls repeat on the same buffers (latency mode, data in L2 as it
    would be right after its producer)."""
    H = synth.FUSED_NORM["hidden"]
    L2 = 126 * 2 ** 20
    for fmt, layout, fname in ((qz.FMT_MXFP8, qz.SF_SWIZZLED, "MXFP8 swizzled"), (qz.FMT_NVFP4, qz.SF_LINEAR, "NVFP4 linear")):
        sweep = []
        for Tn in (tokens or synth.FUSED_NORM["tokens"]):
            qbytes = Tn * (H if fmt == qz.FMT_MXFP8 else H // 2)
            nbytes = Tn * H * 2 * 2 + 2 * H + Tn * H * 2 * 2 + qbytes + qz.sf_bytes(Tn, H, fmt, layout)
            copies = 1 if Tn < 1024 else -(-2 * L2 // nbytes) + 1
            sets = []
            xs, rs, gs = synth.fused_norm_inputs(Tn, device=device)
            for c in range(copies):
                sets.append((xs if c == 0 else xs.clone(), rs if c == 0 else rs.clone(), torch.empty_like(xs),
                             torch.empty_like(xs),
                             torch.empty((Tn, H if fmt == qz.FMT_MXFP8 else H // 2), dtype=torch.uint8, device=device),
                             torch.empty(max(qz.sf_bytes(Tn, H, fmt, layout), 16), dtype=torch.uint8, device=device)))
            amax = torch.tensor([8.0], dtype=torch.float32, device=device) if fmt == qz.FMT_NVFP4 else None
            turn = [0]

            def call():
                x_, r_, y_, h_, q_, sf_ = sets[turn[0] % copies]
                turn[0] += 1
                qz.rmsnorm_quantize(x_, r_, gs, 1e-6, y_, h_, fmt, q_, sf_, layout, amax)

            ms = _time_graph(call, reps=10 * copies) if Tn >= 1024 else _time_graph(call, reps=50)
            sweep.append({"T": Tn, "us": round(ms * 1e3, 2), "GB/s": round(nbytes / (ms / 1e3) / GB, 1),
                          "copies": copies})
            del sets
        big = sweep[-1]
        if big["T"] != 4096:
            big = {"GB/s": 0.0}
        out.append({"workload": f"fused residual+RMSNorm+{fname}, H=7168, T=1..4096 (residual_out written)",
                    "kernel": "rmsnorm_quant_kernel", "sweep": sweep,
                    "timing": "CUDA graph of 50 calls on the same buffers (T < 1024) or of 10 rounds over "
                              "`copies` buffer sets (T >= 1024, inputs larger than L2, no flush)",
                    "frac_of_hbm_peak_T4096": round(big["GB/s"] / peak, 4),
                    "traffic_T4096": ncu_traffic("rmsnorm_quant_kernel") if fmt == qz.FMT_MXFP8 else None})


def _extra_nvfp4_30b(qz, device, rec):
    """One Qwen3-30B-A3B gate_up projection (128 experts of [1536, 2048]) to
    NVFP4 with a per-expert FP32 scale, given and computed, in one call."""
    cfg = synth.QWEN3_30B
    rows, cols = cfg["gate_up"]
    stack = synth.expert_stack(cfg["experts"], (rows, cols), cfg["std"], seed=cfg["seed"], device=device)
    ws = qz.alloc_workspace(cfg["experts"], device)
    for mode, fname, w in ((qz.NVFP4_PER_TENSOR_GIVEN, "given amax", None),
                           (qz.NVFP4_PER_TENSOR_COMPUTE, "computed amax (one cooperative launch)", ws),
                           (qz.NVFP4_PER_TENSOR_COMPUTE, "computed amax (amax pass + quantize pass)", None)):
        ents = qz.alloc_outputs(list(stack.unbind(0)), qz.FMT_NVFP4, qz.SF_SWIZZLED, mode)
        for e in ents:
            e.amax.fill_(0.1)
        tab = qz.ExpertTable(ents)
        ms = _time_graph(lambda m=mode, w=w: qz.quantize_grouped_nvfp4(tab, m, qz.SF_SWIZZLED, workspace=w), reps=5)
        nsf = qz.sf_bytes(rows, cols, qz.FMT_NVFP4, qz.SF_SWIZZLED)
        nbytes = cfg["experts"] * (rows * cols * 2 + rows * cols // 2 + nsf + 4)
        rec(f"Qwen3-30B-A3B gate_up [1536, 2048] x128 experts, NVFP4 {fname}, swizzled, one call", nbytes, ms,
            1 if mode == qz.NVFP4_PER_TENSOR_GIVEN else (2 if w is not None else 3))
        del ents, tab
    del stack
    torch.cuda.empty_cache()


def _extra_large(qz, device, rec, experts=None):
    """One Qwen3-235B-A22B layer: 128 experts per projection per call (or the
    first `experts` of them, for a profiler capture)."""
    cfg = dict(synth.QWEN3_235B)
    if experts:
        cfg["experts"] = experts
    for proj, shape in (("gate_up", cfg["gate_up"]), ("down", cfg["down"])):
        stack = synth.expert_stack(cfg["experts"], shape, cfg["std"], seed=cfg["seed"], device=device)
        rows, cols = shape
        ws = qz.alloc_workspace(cfg["experts"], device)
        for fmt, mode, fname in ((qz.FMT_MXFP8, None, "MXFP8"), (qz.FMT_NVFP4, qz.NVFP4_PER_TENSOR_GIVEN, "NVFP4 given amax"),
                                 (qz.FMT_NVFP4, qz.NVFP4_PER_TENSOR_COMPUTE, "NVFP4 computed amax")):
            ents = qz.alloc_outputs(list(stack.unbind(0)), fmt, qz.SF_SWIZZLED,
                                    mode if mode is not None else qz.NVFP4_PER_ROW)
            if fmt == qz.FMT_NVFP4:
                for e in ents:
                    e.amax.fill_(0.1)
            tab = qz.ExpertTable(ents)
            if fmt == qz.FMT_MXFP8:
                fn = lambda: qz.quantize_grouped_mxfp8(tab, qz.SF_SWIZZLED)  # noqa: E731
            else:
                fn = lambda m=mode: qz.quantize_grouped_nvfp4(  # noqa: E731
                    tab, m, qz.SF_SWIZZLED, workspace=ws if m == qz.NVFP4_PER_TENSOR_COMPUTE else None)
            ms = _time_graph(fn, reps=5)
            nsf = qz.sf_bytes(rows, cols, fmt, qz.SF_SWIZZLED)
            qb = rows * cols if fmt == qz.FMT_MXFP8 else rows * cols // 2
            nbytes = cfg["experts"] * (rows * cols * 2 + qb + nsf + (4 if fmt == qz.FMT_NVFP4 else 0))
            rec(f"Qwen3-235B-A22B {proj} {list(shape)} x{cfg['experts']} experts, {fname}, swizzled", nbytes, ms,
                1 if mode != qz.NVFP4_PER_TENSOR_COMPUTE else 2)
            del ents, tab
        del stack
        torch.cuda.empty_cache()


def _extra_dequant(qz, device, rec):
    """Decode a Qwen3-30B-A3B gate_up projection (128 experts of [1536, 2048])
    back to bf16 from MXFP8 and from NVFP4 (per-tensor scale), in one call."""
    cfg = synth.QWEN3_30B
    rows, cols = cfg["gate_up"]
    stack = synth.expert_stack(cfg["experts"], (rows, cols), cfg["std"], seed=cfg["seed"], device=device)
    for fmt, fname in ((qz.FMT_MXFP8, "MXFP8"), (qz.FMT_NVFP4, "NVFP4 (per-tensor amax)")):
        mode = qz.NVFP4_PER_TENSOR_COMPUTE if fmt == qz.FMT_NVFP4 else qz.NVFP4_PER_ROW
        ents = qz.alloc_outputs(list(stack.unbind(0)), fmt, qz.SF_SWIZZLED, mode)
        tab = qz.ExpertTable(ents)
        if fmt == qz.FMT_MXFP8:
            qz.quantize_grouped_mxfp8(tab, qz.SF_SWIZZLED)
        else:
            qz.quantize_grouped_nvfp4(tab, mode, qz.SF_SWIZZLED)
        ys = torch.empty_like(stack)
        dtab = qz.DqTable([qz.DqEntry(e.q, e.sf, y, e.amax) for e, y in zip(ents, ys.unbind(0))])
        ms = _time_graph(lambda f=fmt, t=dtab: qz.dequantize_grouped(t, f, False, qz.SF_SWIZZLED), reps=5)
        nsf = qz.sf_bytes(rows, cols, fmt, qz.SF_SWIZZLED)
        qb = rows * cols if fmt == qz.FMT_MXFP8 else rows * cols // 2
        nbytes = cfg["experts"] * (qb + nsf + (4 if fmt == qz.FMT_NVFP4 else 0) + rows * cols * 2)
        rec(f"dequantize Qwen3-30B-A3B gate_up [1536, 2048] x128 experts from {fname} to bf16, swizzled, one call",
            nbytes, ms, 1, kernel="dequant_kernel")
        del ents, tab, dtab, ys
    del stack
    torch.cuda.empty_cache()


def _extra_gate_up_split(qz, device, rec):
    """Gate|up split of a folded Qwen3-30B-A3B gate_up projection (128 fused
    experts of [1536, 2048], NVFP4 with a per-tensor amax, swizzled) at row
    768; and the one-pass fold (gate and up quantized straight into their own
    storage, sharing the expert's amax) against fold-then-split."""
    cfg = synth.QWEN3_30B
    rows, cols = cfg["gate_up"]
    E, cut = cfg["experts"], rows // 2
    swz, nv = qz.SF_SWIZZLED, qz.FMT_NVFP4
    stack = synth.expert_stack(E, (rows, cols), cfg["std"], seed=cfg["seed"], device=device)
    nsf, npart = qz.sf_bytes(rows, cols, nv, swz), qz.sf_bytes(cut, cols, nv, swz)
    q = torch.empty((E, rows, cols // 2), dtype=torch.uint8, device=device)
    sf = torch.empty((E, nsf), dtype=torch.uint8, device=device)
    A = torch.empty((E, 1), dtype=torch.float32, device=device)
    fold = qz.ExpertTable([qz.Entry(stack[e], q[e], sf[e], A[e]) for e in range(E)])
    qz.quantize_grouped_nvfp4(fold, qz.NVFP4_PER_TENSOR_COMPUTE, swz)
    qo = torch.empty((E, 2, cut, cols // 2), dtype=torch.uint8, device=device)
    so = torch.empty((E, 2, npart), dtype=torch.uint8, device=device)
    ao = torch.empty((E, 2, 1), dtype=torch.float32, device=device)
    split = qz.SplitTable([qz.SplitEntry(q=q[e], sf=sf[e], rows=rows, cols=cols, cut=cut, sf_out=(so[e, 0], so[e, 1]),
                                         q_out=(qo[e, 0], qo[e, 1]), amax=A[e], amax_out=(ao[e, 0], ao[e, 1]))
                           for e in range(E)])

    def split_call():
        qz.split_fused_experts(split, nv, qz.AMAX_PER_TENSOR, swz, swz)

    ms = _time_graph(split_call, reps=5)
    nbytes = E * (2 * rows * (cols // 2) + nsf + 2 * npart + 3 * 4)
    rec("gate|up split of a folded Qwen3-30B-A3B gate_up projection, 128 fused experts [1536, 2048] NVFP4 swizzled, "
        "cut at row 768, one call", nbytes, ms, 1, kernel="split_fused_kernel", l2="inputs larger than L2",
        traffic=ncu_traffic("split_fused_kernel"))
    parts = qz.ExpertTable([qz.Entry(stack[e, p * cut:(p + 1) * cut], qo[e, p], so[e, p], A[e])
                            for e in range(E) for p in range(2)])
    ms_one = _time_graph(lambda: qz.quantize_grouped_nvfp4(parts, qz.NVFP4_PER_TENSOR_GIVEN, swz), reps=5)
    ms_two = _time_graph(lambda: (qz.quantize_grouped_nvfp4(fold, qz.NVFP4_PER_TENSOR_GIVEN, swz), split_call()),
                         reps=5)
    qbytes = E * (rows * cols * 2 + rows * (cols // 2) + 2 * npart + 4)
    rec("one-pass fold: Qwen3-30B-A3B gate_up [1536, 2048] x128 fused experts quantized to NVFP4 (given shared amax) "
        "straight into separate gate and up storage", qbytes, ms_one, 1, kernel="nvfp4_tile_kernel",
        fold_then_split_us=round(ms_two * 1e3, 2))
    del stack, q, sf, qo, so, fold, split, parts
    torch.cuda.empty_cache()


def _extra_colwise(qz, device, rec):
    """Column-wise (transposed) quantization of a Qwen3-30B-A3B gate_up
    projection (128 experts of [1536, 2048]) to MXFP8 and to NVFP4 (given
    per-tensor amax), swizzled, in one call."""
    cfg = synth.QWEN3_30B
    rows, cols = cfg["gate_up"]
    n = cfg["experts"]
    stack = synth.expert_stack(n, (rows, cols), cfg["std"], seed=cfg["seed"], device=device)
    for fmt, fname in ((qz.FMT_MXFP8, "MXFP8"), (qz.FMT_NVFP4, "NVFP4 (given amax)")):
        qb = rows * cols if fmt == qz.FMT_MXFP8 else rows * cols // 2
        nsf = qz.sf_bytes(cols, rows, fmt, qz.SF_SWIZZLED)
        ents = []
        for x in stack.unbind(0):
            q = torch.empty(qb, dtype=torch.uint8, device=device)
            sf = torch.empty(nsf, dtype=torch.uint8, device=device)
            a = torch.full((1,), 0.1, dtype=torch.float32, device=device) if fmt == qz.FMT_NVFP4 else None
            ents.append(qz.Entry(x, q, sf, a))
        tab = qz.ExpertTable(ents)
        ms = _time_graph(lambda f=fmt, t=tab: qz.quantize_grouped_colwise(t, f, qz.SF_SWIZZLED), reps=5)
        nbytes = n * (rows * cols * 2 + qb + nsf + (4 if fmt == qz.FMT_NVFP4 else 0))
        rec(f"column-wise quantize Qwen3-30B-A3B gate_up [1536, 2048] x128 experts to {fname}, swizzled, one call",
            nbytes, ms, 1, kernel="colwise_kernel")
        del ents, tab
    del stack
    torch.cuda.empty_cache()


def _extra_merge(qz, device, flush, out, peak, tokens=None):
    """Attention decode merge of 8 splits at H = 7168 writing bf16 and MXFP8
    (swizzled) in one kernel, against the same merge writing bf16 followed by
    a standalone MXFP8 quantize of its output; T swept 1..4096."""
    S, H = 8, 7168
    sweep = []
    for Tn in (tokens or (1, 16, 64, 512, 4096)):
        O, lse = synth.merge_partials(S, Tn, H, seed=Tn)
        Od, ld = torch.from_numpy(O).to(device), torch.from_numpy(lse).to(device)
        y = torch.empty((Tn, H), dtype=torch.bfloat16, device=device)
        q = torch.empty((Tn, H), dtype=torch.uint8, device=device)
        sf = torch.empty(max(qz.sf_bytes(Tn, H, qz.FMT_MXFP8, qz.SF_SWIZZLED), 16), dtype=torch.uint8, device=device)
        tab = qz.ExpertTable([qz.Entry(y, q, sf)])

        def fused():
            qz.attention_merge_quantize(Od, ld, y, q, sf, qz.SF_SWIZZLED)

        def unfused():
            qz.attention_merge_quantize(Od, ld, y, None, None, qz.SF_SWIZZLED)
            qz.quantize_grouped_mxfp8(tab, qz.SF_SWIZZLED)

        fl = flush if 512 <= Tn < 2048 else None  # from T = 2048 on the partials alone exceed L2
        reps = 10 if Tn >= 512 else 50
        ms_f = _time_graph(fused, reps=reps, flush=fl)
        ms_u = _time_graph(unfused, reps=reps, flush=fl)
        nbytes = S * Tn * H * 4 + S * Tn * 4 + Tn * H * 2 + Tn * H + qz.sf_bytes(Tn, H, qz.FMT_MXFP8, qz.SF_SWIZZLED)
        sweep.append({"T": Tn, "fused_us": round(ms_f * 1e3, 2), "unfused_us": round(ms_u * 1e3, 2),
                      "fused_GB/s": round(nbytes / (ms_f / 1e3) / GB, 1)})
        del Od, ld, y, q, sf, tab
    big = sweep[-1]
    out.append({"workload": "attention decode merge, 8 splits, H=7168, bf16 + MXFP8 swizzled in one kernel "
                            "vs merge then standalone quantize, T=1..4096",
                "kernel": "attention_merge_kernel", "sweep": sweep,
                "timing": "CUDA graph of 50 calls (T < 512), of 10 calls after an L2 flush each (T = 512), "
                          "or of 10 calls on partials larger than L2 (T >= 2048, no flush)",
                "frac_of_hbm_peak_fused_T4096": round(big["fused_GB/s"] / peak, 4) if big["T"] == 4096 else None})


def _extra_allreduce(qz, device, out, peak, tokens=None, ranks=8):
    """AllReduce epilogue, one-shot form: the sum of 8 rank inputs + residual
    add + RMSNorm + MXFP8 (swizzled), H = 7168, T swept 1..4096.  With one GPU
    the 8 rank inputs are 8 buffers in this GPU's HBM, read through the same
    plain pointers a peer mapping would give: the HBM-side cost of the kernel.
    From T = 1024 on, buffer sets are used round-robin so that a call's bytes
    were last touched more than twice the L2 size ago; below, calls repeat on
    the same buffers."""
    H = synth.FUSED_NORM["hidden"]
    L2 = 126 * 2 ** 20
    fmt, layout = qz.FMT_MXFP8, qz.SF_SWIZZLED
    sweep = []
    for Tn in (tokens or (1, 16, 64, 512, 4096)):
        nbytes = (ranks + 1) * Tn * H * 2 + 2 * H + Tn * H * (2 + 2 + 1) + qz.sf_bytes(Tn, H, fmt, layout)
        copies = 1 if Tn < 1024 else -(-2 * L2 // nbytes) + 1
        xs, r, g = synth.rank_partials(ranks, Tn, device=device)
        sets = []
        for c in range(copies):
            sets.append(([x if c == 0 else x.clone() for x in xs], r if c == 0 else r.clone(),
                         [(torch.empty_like(r), torch.empty_like(r),
                           torch.empty((Tn, H), dtype=torch.uint8, device=device),
                           torch.empty(max(qz.sf_bytes(Tn, H, fmt, layout), 16), dtype=torch.uint8,
                                       device=device))]))
        turn = [0]

        def call():
            xs_, r_, d_ = sets[turn[0] % copies]
            turn[0] += 1
            qz.allreduce_rmsnorm_quantize(xs_, r_, g, 1e-6, d_, fmt, layout, Tn, H)

        ms = _time_graph(call, reps=10 * copies) if Tn >= 1024 else _time_graph(call, reps=50)
        sweep.append({"T": Tn, "us": round(ms * 1e3, 2), "GB/s": round(nbytes / (ms / 1e3) / GB, 1),
                      "bytes_per_call": int(nbytes), "copies": copies})
        del sets, xs, r, g
    big = sweep[-1]
    out.append({"workload": f"AllReduce epilogue (one-shot): sum of {ranks} rank inputs + residual + RMSNorm + "
                            "MXFP8 swizzled, H=7168, T=1..4096 (residual_out written); the rank inputs are "
                            "buffers on this one GPU",
                "kernel": "rmsnorm_quant_kernel_multi", "sweep": sweep,
                "timing": "CUDA graph of 50 calls on the same buffers (T < 1024) or of 10 rounds over "
                          "`copies` buffer sets (T >= 1024, inputs larger than L2, no flush)",
                "frac_of_hbm_peak_T4096": round(big["GB/s"] / peak, 4) if big["T"] == 4096 else None,
                "traffic_T4096": ncu_traffic("rmsnorm_quant_kernel_multi")})


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------

def allreduce_nvlink(qz, device, rank, world, tokens=(16, 512, 4096)):
    """The AllReduce epilogue across the ranks' GPUs (only under torchrun,
    N > 1): every rank's buffer is mapped into every process through CUDA IPC
    (PeerBuffers), the rank inputs are read and the destinations written with
    plain peer loads and stores over NVLink (no multicast), and each call sits
    between two stream-ordered NCCL barriers.  CUDA events bracket the kernel
    alone on each rank; the time is the max over ranks.  The NVLink bound of a
    call is the bytes that must cross it (one-shot: (n - 1) T H 2 reads per
    rank; slice form: (n - 1)/n of them plus (n - 1)/n of the outputs written
    to peers) over the measured 770 GB/s peer copy per direction."""
    from nvfp4_quantization_moe_b200 import allreduce as ar
    H = synth.FUSED_NORM["hidden"]
    fmt, layout = qz.FMT_MXFP8, qz.SF_SWIZZLED
    Tmax = max(tokens)
    L = ar.SymmetricLayout(Tmax, H, fmt, layout)
    buf = torch.zeros(L.total, dtype=torch.uint8, device=device)
    xs, r, g = synth.rank_partials(world, Tmax, device=device)
    buf[L.x:L.x + Tmax * H * 2].view(torch.bfloat16).view(Tmax, H).copy_(xs[rank])
    one = torch.ones(1, dtype=torch.int32, device=device)

    def barrier():
        torch.distributed.all_reduce(one, op=torch.distributed.ReduceOp.MAX)  # every rank's prior stream work is done

    timed = []

    def launch(*a, **kw):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qz.allreduce_rmsnorm_quantize(*a, **kw)
        e1.record()
        timed.append((e0, e1))

    out = {"ranks": world, "H": H, "format": "MXFP8 swizzled, residual_out written", "sweep": []}
    with ar.PeerBuffers(buf.data_ptr()) as pb:
        for slice_form in (False, True):
            ep = ar.AllReduceEpilogue(rank, world, pb.bases, L, barrier, slice_form=slice_form, launch=launch)
            for T in tokens:
                for _ in range(3):
                    ep(T, r[:T], g, 1e-6)
                torch.cuda.synchronize()
                timed.clear()
                for _ in range(10):
                    ep(T, r[:T], g, 1e-6)
                torch.cuda.synchronize()
                us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in timed)
                us = max_over_ranks([us], device)[0]
                rows = T if not slice_form else ar.rank_rows(T, world, rank)[1] - ar.rank_rows(T, world, rank)[0]
                bf = T * H * 2
                remote_in = (world - 1) * bf if not slice_form else (world - 1) * rows * H * 2
                outs = rows * H * (2 + 2 + 1) + qz.sf_bytes(rows, H, fmt, layout)
                remote_out = 0 if not slice_form else (world - 1) * outs
                nvl = remote_in + remote_out
                out["sweep"].append({"form": "slice" if slice_form else "one-shot", "T": T, "us": round(us, 2),
                                     "nvlink_bytes": int(nvl), "nvlink_GB/s": round(nvl / (us / 1e3) / GB, 1),
                                     "frac_of_770": round(nvl / (us / 1e3) / GB / 770.0, 4)})
        torch.cuda.synchronize()
        torch.distributed.barrier()
    del buf
    return out


def oracle_prequant_sample(threads: int, target_s: float = 10.0, min_pairs: int = 1, pairs: int = 0):
    """Time the CPU oracle on a bounded sample of the headline workload: whole
    Qwen3-235B-A22B experts (one gate_up [3072, 4096] and one down
    [4096, 1536]) each quantized to MXFP8, to NVFP4 with the amax computed and
    to NVFP4 with it given -- the six calls of a layer, per expert pair --
    repeated over ``threads`` host threads for about ``target_s`` seconds.
    ``pairs`` > 0 skips the sizing run.  Returns (GB/s, threads, sample
    description, seconds, pairs)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    cfg = synth.QWEN3_235B
    xs = {p: synth.bf16_bits(synth.moe_layer(dict(cfg, experts=1), 0, p, device="cpu")[0]) for p in PROJS}
    per_pair = 0
    for p in PROJS:
        r, c = cfg[p]
        per_pair += r * c * 2 + r * c + (r * c // 32)                      # MXFP8 (no padding at these shapes)
        per_pair += 2 * (r * c * 2 + r * c // 2 + (r * c // 16) + 4)      # NVFP4 computed, NVFP4 given

    def pair(_):
        for p in PROJS:
            x = xs[p]
            oracle.quantize_mxfp8(x, oracle.SWIZZLED)
            _, _, a = oracle.quantize_nvfp4(x, oracle.SWIZZLED, oracle.NVFP4_PER_TENSOR_COMPUTE)
            oracle.quantize_nvfp4(x, oracle.SWIZZLED, oracle.NVFP4_PER_TENSOR_GIVEN, float(a[0]))

    if pairs <= 0:
        t0 = time.perf_counter()
        pair(0)
        one = time.perf_counter() - t0
        pairs = max(min_pairs, threads, int(round(target_s / max(one, 1e-3) * threads)))
    t0 = time.perf_counter()
    if threads <= 1:
        for i in range(pairs):
            pair(i)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(pair, range(pairs)))
    dt = time.perf_counter() - t0
    nbytes = pairs * per_pair
    desc = (f"{pairs} x (gate_up [3072,4096] + down [4096,1536]) Qwen3-235B-A22B experts, each to MXFP8, NVFP4 "
            f"computed amax and NVFP4 given amax (swizzled), {nbytes / GB:.2f} GB, {threads} thread(s)")
    return nbytes / dt / GB, threads, desc, dt, pairs


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands on the host cores, on
    the headline's workload (a bounded sample per step), rank 0 only."""
    if rank != 0:
        return
    import oracle
    threads = oracle.host_threads()
    vals, t_total, desc = [], 0.0, None
    npairs = 0
    for i in range(args.warmup + args.steps):
        # the first step sizes the sample, the others repeat it
        v, _, desc, dt, npairs = oracle_prequant_sample(
            threads, target_s=max(1.0, 60.0 / max(1, args.steps + args.warmup)), pairs=npairs)
        if i >= args.warmup:
            vals.append(v)
            t_total += dt
    value = statistics.median(vals)
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t_total / max(1, args.steps), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16->mxfp8/nvfp4 (f32 host)", "data": "synthetic", "impl": "reference",
            "config": {"workload": HEADLINE_WORKLOAD, "sample": desc},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


HEADLINE_WORKLOAD = "Qwen3-235B-A22B prequant: 94 layers x 2 projections x 128 experts, MXFP8 + NVFP4 (computed, given)"


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------

def refit_30b(qz, device, args, rank, dist_ok, peak):
    """The Qwen3-30B-A3B MXFP8 refit step (config 2): 48 layers resident,
    16 experts per call, calls round-robin on two streams; the same steps in
    order on one stream give each launch's own event time."""
    work = Refit30B(qz, device, layers=args.layers, seed_offset=rank)
    side = [torch.cuda.Stream() for _ in range(args.streams)] if args.streams > 1 else None
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    total_ms, _, _ = time_steps(work, args.steps, args.warmup, stream, dist_ok, side=side, per_launch=False)
    single_ms, single_launch_ms, _ = time_steps(work, args.steps, 1, stream, dist_ok)
    indep_ms, _, _ = time_steps(work, args.steps, 1, stream, dist_ok, per_launch=False, independent=True)
    total_ms, single_ms, indep_ms = max_over_ranks([total_ms, single_ms, indep_ms], device)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    value = aggregate_gbs(work.bytes, world, args.steps, total_ms)
    call_bytes = [b for _, b in work.calls] * args.steps
    achieved = sum(call_bytes) / (total_ms / 1e3) / GB
    achieved_single = sum(call_bytes) / (sum(single_launch_ms) / 1e3) / GB
    out = {"value": round(value, 1), "unit": "GB/s", "ms_per_step": round(total_ms / args.steps, 3),
           "frac": round(achieved / peak, 4), "kernel": work.kernel,
           "workload": f"Qwen3-30B-A3B MXFP8 refit: {args.layers} layers x 128 experts, 16 experts/call, swizzled",
           "bytes_per_step_per_gpu": work.bytes, "launches_per_step": work.launches,
           "issue": f"calls round-robin on {args.streams} streams" if side else "calls in order on one stream",
           "bytes_per_launch": int(np.mean([b for _, b in work.calls])),
           "effective_launch_us": round(1e3 * total_ms / (work.launches * args.steps), 2),
           "traffic": ncu_traffic(work.kernel, "qwen3-30b-refit"),
           "single_stream": {"value": round(aggregate_gbs(work.bytes, world, args.steps, single_ms), 1),
                             "frac": round(achieved_single / peak, 4),
                             "mean_launch_us": round(1e3 * float(np.mean(single_launch_ms)), 2)},
           "single_stream_independent": {
               "value": round(aggregate_gbs(work.bytes, world, args.steps, indep_ms), 1),
               "frac": round(sum(call_bytes) / (indep_ms / 1e3) / GB / peak, 4),
               "how": "calls in order on one stream, each declared QZ_OPT_INDEPENDENT (programmatic dependent "
                      "launch overlaps each call's tail with the next call's tiles); region timed"}}
    del work
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: 94 for the Qwen3-235B-A22B sweep, 48 for the 30B refit)")
    ap.add_argument("--streams", type=int, default=2, help="streams the independent 30B refit calls are spread over")
    ap.add_argument("--compute-path", choices=["single", "three"], default="single",
                    help="NVFP4 computed amax: one cooperative launch with a workspace, or clear + amax + quantize")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-refit", action="store_true", help="skip the Qwen3-30B-A3B refit step")
    ap.add_argument("--no-allreduce", action="store_true",
                    help="with N > 1: skip the AllReduce epilogue across the ranks' GPUs")
    ap.add_argument("--config", type=int, choices=[1, 2, 3, 4, 5], default=None,
                    help="one of the five workloads: 1 tiny MXFP8 group (latency), 2 the Qwen3-30B-A3B refit step, "
                         "3 the row-scaled NVFP4 split activation, 4 the fused residual + RMSNorm sweep, 5 the "
                         "Qwen3-235B-A22B sweep (the default run)")
    ap.add_argument("--only", choices=["tiny", "split", "fused", "nvfp4", "large", "dequant", "merge", "colwise",
                                       "gateup", "allreduce"],
                    default=None,
                    help="time only this secondary workload and print its record (profiling aid)")
    ap.add_argument("--experts", type=int, default=None,
                    help="experts per call of the Qwen3-235B-A22B extra workload (fewer for a profiler capture)")
    ap.add_argument("--tokens", type=str, default=None,
                    help="comma-separated token counts for the fused, merge and AllReduce sweeps")
    args = ap.parse_args()
    if args.config in (1, 3, 4):
        args.only = {1: "tiny", 3: "split", 4: "fused"}[args.config]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_ok = world > 1

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import nvfp4_quantization_moe_b200 as qz
    qz.load()
    assert torch.cuda.is_available(), "bench.py --impl ours needs a CUDA device"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if dist_ok:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    stream = torch.cuda.current_stream()
    peak, peak_kind = hbm_peak()
    if args.only:
        toks = [int(t) for t in args.tokens.split(",")] if args.tokens else None
        print(json.dumps({"only": args.only,
                          "extra": extra_workloads(qz, device, stream, peak, (args.only,), toks, args.experts)}))
        return

    if args.config == 2:
        # the 30B refit step as the headline
        args.layers = args.layers or 48
        with ClockSampler(local) as clocks:
            r = refit_30b(qz, device, args, rank, dist_ok, peak)
        line = {"metric": METRIC, "value": r["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16->mxfp8 (e4m3 + e8m0)", "data": "synthetic",
                "config": {"workload": r["workload"], "l2": "inputs larger than L2",
                           "parallelism": f"{world} independent replicas (weak scaling, no collective)"},
                "roofline": {"bound": "hbm", "achieved": round(r["frac"] * peak, 1), "peak": peak, "unit": "GB/s",
                             "frac": r["frac"], "traffic": r["traffic"], "kernel": r["kernel"],
                             "single_stream_frac": r["single_stream"]["frac"]},
                "clocks": clocks.summary(), "gpu_launches": r["launches_per_step"] * (args.steps + 1),
                "refit_30b": r}
        if dist_ok:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return

    # ---- default: the Qwen3-235B-A22B sweep (config 5) ----
    refit = None
    if args.config is None and not args.no_refit:
        refit_args = argparse.Namespace(**vars(args))
        refit_args.layers = 48
        refit_args.steps, refit_args.warmup = min(args.steps, 10), min(args.warmup, 3)
        refit = refit_30b(qz, device, refit_args, rank, dist_ok, peak)
    layers = args.layers or synth.QWEN3_235B["layers"]
    work = Prequant235B(qz, device, layers=layers, rank=rank, compute_workspace=args.compute_path == "single")
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        per, total_ms, sweep_ms = time_sweep(work, args.steps, args.warmup, stream, dist_ok)
    total_ms, sweep_ms = max_over_ranks([total_ms, sweep_ms], device)
    value = aggregate_gbs(work.bytes, world, args.steps, total_ms)
    roof = sweep_roofline(per, peak, peak_kind, {"nvfp4_compute": work.compute_launches}, work.kernels)
    launches = work.launches_per_layer * layers * args.steps
    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16->mxfp8/nvfp4 (e4m3+e8m0, e2m1+e4m3+f32)",
            "data": "synthetic",
            "frac_of_hbm_peak": round(value / world / peak, 4),
            "config": {"workload": HEADLINE_WORKLOAD,
                       "experts": "gate_up [3072,4096] + down [4096,1536] bf16 N(0,0.02), seed 5+layer",
                       "calls": "6 per layer: MXFP8, NVFP4 amax computed, NVFP4 amax given; 128 experts each",
                       "layers_per_step": layers, "bytes_per_step_per_gpu": work.bytes,
                       "l2": "inputs larger than L2 (3.2 / 1.6 GB per call)",
                       "timing": "sum of per-call CUDA events; layer regeneration untimed",
                       "compute_path": "one cooperative launch" if args.compute_path == "single" else "three launches",
                       "parallelism": f"{world} independent replicas (weak scaling, no collective)"},
            "roofline": roof, "clocks": clocks.summary(), "gpu_launches": launches,
            "sweep_device_ms_per_step": round(sweep_ms / args.steps, 1)}
    if refit is not None:
        line["refit_30b"] = refit
    del work
    torch.cuda.empty_cache()

    if dist_ok and not args.no_allreduce:
        try:
            line["allreduce_nvlink"] = allreduce_nvlink(qz, device, rank, world)
        except Exception as exc:  # reported, never allowed to void the measured line
            line["allreduce_nvlink"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    if rank == 0 and not args.no_e2e:
        line["e2e"] = e2e_prequant(qz, device, steps=2, warmup=1, compute_workspace=args.compute_path == "single")
    if rank == 0 and not args.no_extra and args.config is None:
        line["extra"] = extra_workloads(qz, device, stream, peak,
                                        which=("tiny", "split", "fused", "nvfp4", "dequant", "merge", "colwise",
                                               "gateup", "allreduce"))
    if rank == 0 and not args.no_cpu:
        import oracle
        threads = oracle.host_threads()
        v1, _, d1, t1, _ = oracle_prequant_sample(1, target_s=8.0)
        vn, cores, dn, tn, _ = oracle_prequant_sample(threads, target_s=10.0)
        line["cpu_baseline"] = {"value": round(vn, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": dn, "seconds": round(tn, 2),
                                "single_thread": {"value": round(v1, 4), "unit": "GB/s", "cores": 1, "sample": d1,
                                                  "seconds": round(t1, 2)}}
    if dist_ok:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
