#!/usr/bin/env python
"""Benchmark of the MSDeformAttn core on B200: one step = the fused forward
(softmax, location map, bilinear gather; it also writes the locations and
weights the backward needs) followed by the backward (grad_value scatter,
grad_sampling_locations, grad_attention_weights) over one batch of the chosen
synthetic workload.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload encoder]
  python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Timing: W untimed warm-up steps; then K steps, each preceded by an L2 flush
(a memset of twice the L2 size, outside the timed events), each timed with
CUDA events on the launching stream; the K-step region is bracketed by a
barrier and torch.cuda.synchronize() on both sides; the reported time is the
max over ranks.  Multi-GPU: every rank runs its own batch (weak scaling; the
batch entries are independent, so there is no data-path collective).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from scale_deformable_attention_02_b200 import workloads as wl  # noqa: E402

METRIC = "MSDeformAttn fwd+bwd queries/sec and effective HBM GB/s (% roofline) on 1 B200"
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_TEXT = {
    "encoder": "encoder-shaped fused fwd+bwd, fp32 value: N=2, Lq=S=17821 (one query per "
               "pixel of 100x134, 50x67, 25x34, 13x17), M=8, D=32, L=4, K=4",
    "encoder_bf16": "encoder-shaped fused fwd+bwd, bf16 value, fp32 accumulation: N=2, "
                    "Lq=S=17821, M=8, D=32, L=4, K=4",
    "stress": "high-resolution stress fused fwd+bwd, bf16 value, fp32 accumulation: N=8, "
              "Lq=S=37150 (167x167, 84x84, 42x42, 21x21), M=8, D=32, L=4, K=8, 5% of "
              "samples pushed out of range",
    "decoder": "decoder-shaped fused fwd+bwd, fp32 value: N=2, Lq=300, M=8, D=32, L=4, K=4, "
               "S=17821",
    "encoder_compass": "encoder-shaped fused fwd+bwd at the compass initialisation (head m "
                       "samples k px along direction m on every level, uniform weights), "
                       "fp32 value: N=2, Lq=S=17821, M=8, D=32, L=4, K=4",
}


# ---------------------------------------------------------------------------
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_TEXT), default="encoder")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle leg")
    # the pipelined e2e steps: filling and draining the copy-in / compute /
    # copy-out pipeline costs about one download, spread over these steps
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--no-floors", action="store_true",
                    help="skip the memory-floor replay of the workload's corner rows")
    ap.add_argument("--graph", action="store_true",
                    help="capture the forward and the backward as two CUDA graphs and time "
                         "their replays (the launch-latency path for small problems such "
                         "as the decoder)")
    ap.add_argument("--schedule", choices=["tiled", "untiled"], default=None,
                    help="untiled: the msda.h calls (default); tiled: tile plan + msda_tiled.h "
                         "calls")
    ap.add_argument("--halo", type=int, default=None,
                    help="window halo of the tiled schedule, pixels (default per workload)")
    ap.add_argument("--ctas-per-sm", type=int, default=None,
                    help="resident CTAs the tiled windows are sized for (default per workload)")
    ap.add_argument("--also", default="encoder_bf16,stress",
                    help="comma-separated workloads timed briefly after the main one and "
                         "reported under 'also' (rank 0, one GPU); empty for none")
    ap.add_argument("--also-steps", type=int, default=5)
    ap.add_argument("--step", choices=["split", "fused"], default="split",
                    help="split: fused forward writing locations and weights, then "
                         "msda_backward (grad value, locations, weights); fused: fused "
                         "forward writing only out, then msda_backward_fused (grad value, "
                         "reference points, offsets, logits)")
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_workload(name: str, rank: int) -> wl.Workload:
    """Rank r's own batch: the same shapes, its own seed (weak scaling)."""
    w = wl.WORKLOADS[name]
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(vals, world: int, device):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# ---------------------------------------------------------------------------
# algorithmic (unique) bytes per launch
# ---------------------------------------------------------------------------
def algorithmic_bytes(w: wl.Workload, step: str = "split", touched_rows=None) -> dict:
    """Minimum HBM traffic of each launch: every input read once, every
    output written once.  The value map counts once per (pixel, head) row
    that some sample touches (all rows when touched_rows is None), although
    its rows are gathered many times; grad_value is an output of every row;
    the backward's zero-fill of it is not counted.  split: the forward also
    writes locations and weights, which the backward reads; fused: neither
    pass stores them."""
    N, Lq, S, M, D, L, K = (w.N, w.queries, w.S, w.M, w.D, w.L, w.K)
    esz = 2 if w.value_dtype == "bf16" else 4
    samples = N * Lq * M * L * K
    value = (N * S * M if touched_rows is None else touched_rows) * D * esz
    gvalue = N * S * M * D * 4
    ref = N * Lq * 2 * 4
    outb = N * Lq * M * D * 4
    per = samples * 12  # (x, y) and one weight/logit per sample, fp32
    if step == "fused":
        fwd = value + ref + per + outb
        bwd = value + ref + per + outb + gvalue + ref + per
    else:
        fwd = value + ref + per + outb + per
        bwd = value + per + outb + gvalue + per
    return {"fwd": fwd, "bwd": bwd, "samples": samples}


# Device sources behind each schedule's kernels (the tiled kernels include the
# untiled ones' helpers).
UNTILED_SOURCES = ("msda_fwd.cu", "msda_bwd.cu", "msda_common.cuh", "msda_rows.cuh",
                   "msda_types.h")
TILED_SOURCES = UNTILED_SOURCES + ("msda_fwd_tiled.cu", "msda_bwd_tiled.cu",
                                   "msda_tile_plan.cu", "msda_tile.cuh", "msda_tma.cuh")


def kernel_source_hash(schedule: str = "untiled") -> str:
    """sha256 of one schedule's forward and backward device code: the kernel
    sources and device headers and the launch-parameter structs, with comments
    and blank space removed, so that a counter taken on those kernels stays
    valid across edits that do not touch them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scale_deformable_attention_02_b200", "csrc")

    def norm(text):
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        return " ".join(text.split())

    tiled = schedule == "tiled"
    for f in TILED_SOURCES if tiled else UNTILED_SOURCES:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + norm(fh.read()).encode())
    with open(os.path.join(csrc, "msda_internal.h"), encoding="utf-8") as fh:
        internal = norm(fh.read())
    structs = ("FwdParams", "BwdParams") + (
        ("TileView", "FwdTiledParams", "BwdTiledParams") if tiled else ())
    for name in structs:
        m = re.search(r"struct " + name + r" \{.*?\};", internal)
        h.update(name.encode() + b"\0" + (m.group(0) if m else "").encode())
    return h.hexdigest()


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_key(workload: str, step: str, schedule: str) -> str:
    """Entry of profiles/traffic.json for a bench configuration: the workload,
    "/fused" for the fused step, "/tiled" for the tiled kernels."""
    key = workload if step == "split" else workload + "/fused"
    return key + "/tiled" if schedule == "tiled" else key


def read_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[workload][kernel]
        schedule = "tiled" if workload.endswith("/tiled") else "untiled"
        if e.get("source_sha256") != kernel_source_hash(schedule):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, pci_bus_id: str | None, fallback_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = None
            if pci_bus_id:
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByPciBusId(pci_bus_id.encode())
                except Exception:
                    self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(fallback_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self.nvml = None
            self.error = repr(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
                return
            time.sleep(self.period)

    def start(self):
        if self.nvml is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": self.error or "no samples"}
        mhz = [s[1] for s in self.samples]
        active = 0
        for s in self.samples:
            active |= s[2]
        reasons = [k for k, bit in self.REASONS.items() if active & bit and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "sm_mhz_min": min(mhz), "source": "NVML, every 2 ms during the timed steps"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
# Window halo of the tiled schedule per workload: about twice the standard
# deviation of the workload's offsets (the window-hit replay in the design doc), at
# least 3 pixels; the compass offsets reach K = 4 pixels.
TILE_HALO = {"encoder": 3, "encoder_bf16": 3, "encoder_compass": 4, "stress": 8, "decoder": 4,
             "tiny": 1}
# Resident CTAs per SM the tiled windows are sized for.
TILE_CTAS = {"stress": 1}
# Default schedule: untiled (the msda.h calls).  The tiled schedule
# (msda_tiled.h) stages value windows in shared memory and cuts the L2->SM
# bytes and the L2 reductions, but measured slower on B200 for every workload
# here (encoder fp32: forward 202 against 163 us, backward 693 against
# 439 us); it stays selectable with --schedule tiled.
DEFAULT_SCHEDULE = "untiled"


class Steps:
    """Device tensors of one workload and its forward and backward calls.
    `schedule` tiled: the step rebuilds the tile plan from the reference
    points (msda_tile_plan_build), then runs the tiled forward and backward;
    untiled: the msda.h calls.  `step` split: the fused forward writes the
    locations and weights, msda_backward reads them; fused: the forward
    writes only out, msda_backward_fused recomputes them."""

    def __init__(self, torch, device, w, inp, step, schedule, halo=None, ctas=None):
        import scale_deformable_attention_02_b200 as m
        self.m, self.w, self.step, self.schedule = m, w, step, schedule
        self.sh = inp["spatial_shapes"]
        self.starts, _ = m.msda_level_start_index(self.sh)

        def dev_tensor(a):
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
            return torch.from_numpy(a).to(device)

        self.value = dev_tensor(inp["value"])
        self.ref = dev_tensor(inp["reference_points"])
        self.off = dev_tensor(inp["offsets"])
        self.logits = dev_tensor(inp["logits"])
        self.gout = dev_tensor(inp["grad_out"])
        self.out = torch.empty((w.N, w.queries, w.M * w.D), device=device)
        self.loc = torch.empty_like(self.off)
        self.attn = torch.empty_like(self.logits)
        self.gval = torch.empty((w.N, w.S, w.M, w.D), device=device)
        self.gloc = torch.empty_like(self.off)
        self.gattn = torch.empty_like(self.logits)
        self.gref = torch.empty_like(self.ref)
        self.plan = None
        if schedule == "tiled":
            self.halo = TILE_HALO.get(w.name, 3) if halo is None else halo
            self.ctas = TILE_CTAS.get(w.name, 2) if ctas is None else ctas
            self.plan = m.msda_tile_plan(self.value, self.sh, self.starts, self.ref, K=w.K,
                                         halo=self.halo, ctas_per_sm=self.ctas)
        # our kernels per step: (plan build,) forward, backward
        self.launches = 3 if schedule == "tiled" else 2

    def describe(self) -> dict:
        if self.plan is None:
            return {"schedule": "untiled (msda.h calls)"}
        gx, gy = self.plan.grid
        return {"schedule": "tiled (msda_tiled.h): the tile plan is rebuilt from the reference "
                            "points inside every timed forward",
                "halo_px": self.halo, "ctas_per_sm": self.ctas, "grid": [gx, gy],
                "windows": self.plan.windows, "window_kb": self.plan.desc.window_bytes / 1024}

    def kernel_names(self) -> dict:
        if self.plan is not None:
            f = ("tile_plan_kernel + fwd_tiled_kernel (msda_tile_plan_build + "
                 "msda_forward_fused_tiled)")
            b = ("memset + bwd_tiled_kernel (msda_backward_fused_tiled)" if self.step == "fused"
                 else "memset + bwd_tiled_kernel (msda_backward_tiled)")
        else:
            f = "fwd_kernel (msda_forward_fused)"
            b = ("memset + bwd_kernel (msda_backward_fused)" if self.step == "fused"
                 else "memset + bwd_kernel (msda_backward)")
        return {"fwd": f, "bwd": b}

    # stream=None: the current stream (the capture stream while a graph records)
    def fwd(self, st, t=None):
        m, t = self.m, t or self
        extra = {} if self.step == "fused" else {"sampling_locations_out": t.loc,
                                                  "attention_weights_out": t.attn}
        if self.plan is not None:
            m.msda_tile_plan_rebuild(self.plan, t.ref, buffer=getattr(t, "plan_buf", None),
                                     stream=st)
            plan = self.plan if not hasattr(t, "plan_buf") else \
                m.TilePlan(self.plan.desc, t.plan_buf)
            m.msda_forward_fused_tiled(t.value, self.sh, self.starts, t.ref, t.off, t.logits,
                                       plan, out=t.out, stream=st, **extra)
        else:
            m.msda_forward_fused(t.value, self.sh, self.starts, t.ref, t.off, t.logits,
                                 out=t.out, stream=st, **extra)

    def bwd(self, st, t=None):
        m, t = self.m, t or self
        sh, starts = self.sh, self.starts
        plan = None
        if self.plan is not None:
            plan = self.plan if not hasattr(t, "plan_buf") else \
                m.TilePlan(self.plan.desc, t.plan_buf)
        if self.step == "fused":
            kw = dict(grad_value=t.gval, grad_reference_points=t.gref, grad_offsets=t.gloc,
                      grad_logits=t.gattn, stream=st)
            if plan is not None:
                m.msda_backward_fused_tiled(t.value, sh, starts, t.ref, t.off, t.logits, t.gout,
                                            plan, **kw)
            else:
                m.msda_backward_fused(t.value, sh, starts, t.ref, t.off, t.logits, t.gout, **kw)
        else:
            kw = dict(grad_value=t.gval, grad_sampling_locations=t.gloc,
                      grad_attention_weights=t.gattn, stream=st)
            if plan is not None:
                m.msda_backward_tiled(t.value, sh, starts, t.loc, t.attn, t.gout, plan, **kw)
            else:
                m.msda_backward(t.value, sh, starts, t.loc, t.attn, t.gout, **kw)


def time_steps(torch, steps, stream, flush, K, warmup, clocks=None):
    """K timed steps after `warmup` untimed ones, each after an L2 flush:
    per-step (fwd, bwd, step) milliseconds from CUDA events on `stream`."""
    for _ in range(warmup):
        flush.zero_()
        steps.fwd(stream)
        steps.bwd(stream)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        steps.fwd(stream)
        ev[i][1].record(stream)
        steps.bwd(stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.stop()
    return ([ev[i][0].elapsed_time(ev[i][1]) for i in range(K)],
            [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)],
            [ev[i][0].elapsed_time(ev[i][2]) for i in range(K)])


def sub_record(torch, device, name, args, flush, peak, peak_kind):
    """Device timing of another workload in the same run (a few steps): the
    forward and backward times, queries/s, HBM fractions and clocks."""
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w)
    sched = args.schedule or DEFAULT_SCHEDULE
    st = Steps(torch, device, w, inp, "split", sched)
    del inp
    stream = torch.cuda.current_stream(device)
    clocks = ClockSampler(_pci_bus_id(torch, device), _nvml_index(device.index or 0))
    f, b, s = time_steps(torch, st, stream, flush, args.also_steps, 3, clocks)
    ab = algorithmic_bytes(w, "split")
    ms_f, ms_b, ms_s = statistics.fmean(f), statistics.fmean(b), statistics.fmean(s)
    rec = {"workload": WORKLOAD_TEXT[name], "value_dtype": w.value_dtype, "steps": len(s),
           "warmup": 3, "ms_per_step": ms_s, "queries_per_s": w.N * w.queries / (ms_s / 1e3),
           "fwd_ms": ms_f, "bwd_ms": ms_b,
           "fwd_algorithmic_bytes": ab["fwd"], "bwd_algorithmic_bytes": ab["bwd"],
           "fwd_frac_of_" + peak_kind: ab["fwd"] / (ms_f / 1e3) / 1e9 / peak,
           "bwd_frac_of_" + peak_kind: ab["bwd"] / (ms_b / 1e3) / 1e9 / peak,
           "kernels": st.kernel_names(), "clocks": clocks.summary(), **st.describe()}
    del st
    torch.cuda.empty_cache()
    return rec


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=device)
    w = rank_workload(args.workload, rank)
    inp = wl.make_inputs(w)
    schedule = args.schedule or DEFAULT_SCHEDULE
    st = Steps(torch, device, w, inp, args.step, schedule, args.halo, args.ctas_per_sm)
    sched_desc = st.describe()
    sh, starts = st.sh, st.starts
    value, ref, off, logits = st.value, st.ref, st.off, st.logits
    stream = torch.cuda.current_stream(device)

    graphs = []
    timed = st
    if args.graph:
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):  # first launches (occupancy queries) off the capture
            st.fwd(None)
            st.bwd(None)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        gf, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gf):
            st.fwd(None)
        with torch.cuda.graph(gb):
            st.bwd(None)
        graphs = [gf, gb]

        class Replay:
            def fwd(self, s):
                gf.replay()

            def bwd(self, s):
                gb.replay()
        timed = Replay()

    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 64 << 20), dtype=torch.uint8, device=device)

    K = args.steps
    clocks = ClockSampler(_pci_bus_id(torch, device), _nvml_index(local))
    if world > 1:
        dist.barrier()
    fwd_ms, bwd_ms, step_ms = time_steps(torch, timed, stream, flush, K, args.warmup, clocks)
    if world > 1:
        dist.barrier()
    ms_step, ms_fwd, ms_bwd = max_over_ranks(
        [statistics.fmean(step_ms), statistics.fmean(fwd_ms), statistics.fmean(bwd_ms)],
        world, device)
    queries = w.N * w.queries
    value_qps = queries * world / (ms_step / 1e3)

    # ---- end to end through the binding with host buffers -----------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, torch, dist, world, device, stream, inp, w, st)

    # ---- roofline of the dominant launch ----------------------------------
    offs = corner_rows(torch, w, sh, starts, value, ref, off, logits)
    touched = int(torch.unique(offs).numel())
    peak, peak_kind = read_peaks()
    ab = algorithmic_bytes(w, args.step, touched)
    dom = "bwd" if ms_bwd >= ms_fwd else "fwd"
    dom_ms = ms_bwd if dom == "bwd" else ms_fwd
    achieved = ab[dom] / (dom_ms / 1e3) / 1e9
    names = st.kernel_names()
    kernels = {
        "fwd": {"kernel": names["fwd"], "ms": ms_fwd, "algorithmic_bytes": ab["fwd"],
                "GB_s": ab["fwd"] / (ms_fwd / 1e3) / 1e9},
        "bwd": {"kernel": names["bwd"], "ms": ms_bwd, "algorithmic_bytes": ab["bwd"],
                "GB_s": ab["bwd"] / (ms_bwd / 1e3) / 1e9},
    }
    for k in kernels.values():
        k["frac_of_" + peak_kind] = k["GB_s"] / peak
    tkey = traffic_key(args.workload, args.step, schedule)
    roofline = {
        "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
        "frac": achieved / peak, "frac_of_nominal_8000": achieved / 8000.0,
        "value_rows_touched": touched, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
        if peak_kind == "measured" else "fallback 6.65 TB/s",
        "traffic": read_traffic(tkey, dom),
        "kernel": kernels[dom]["kernel"],
        "algorithmic_bytes_per_launch": ab[dom],
    }

    floors = None
    if not args.no_floors:
        floors = memory_floors(torch, w, offs, value, flush)
        if floors:
            kernels["fwd"]["frac_of_row_floor"] = floors["gather_us"] / (ms_fwd * 1e3)
            kernels["bwd"]["frac_of_row_floor"] = floors["gather_reduce_us"] / (ms_bwd * 1e3)
    del offs

    also = []
    if rank == 0 and world == 1 and args.also:
        del st, inp
        torch.cuda.empty_cache()
        for name in args.also.split(","):
            if name and name != args.workload:
                also.append(sub_record(torch, device, name, args, flush, peak, peak_kind))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, wl.make_inputs(w))

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value_qps,
            "unit": "queries/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded numpy PCG64; shapes of the Deformable DETR "
                    "encoder/decoder, no dataset or trained weights)",
            "config": {
                "workload": WORKLOAD_TEXT[args.workload],
                "step": ("fused forward (out only) + fused backward (grad value, reference "
                         "points, offsets, logits)" if args.step == "fused" else
                         "fused forward (out, locations, weights) + backward (grad value, "
                         "locations, weights)"),
                "value_dtype": w.value_dtype,
                "global_batch": w.N * world,
                "queries_per_step": queries * world,
                "parallelism": f"dp{world} (independent batches, no collective)",
                "l2": "flushed before every timed step (memset of 2x L2, outside the events)",
                "launch": ("two CUDA graph replays per step (forward graph, backward graph)"
                           if args.graph else "eager launches through the binding"),
                **sched_desc,
            },
            "effective_GB_s": (ab["fwd"] + ab["bwd"]) / (ms_step / 1e3) / 1e9,
            "kernels": kernels,
            "roofline": roofline,
            "row_floors": floors,
            "also": also,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step(schedule) * K,
            "clocks": clocks.summary(),
            "impl": "ours",
        }
        print(json.dumps(line), flush=True)
    del graphs
    if world > 1:
        dist.destroy_process_group()


def launches_per_step(schedule: str) -> int:
    """Our kernels in one step: (the tile plan's sort,) the forward and the
    backward; the backward's zero-fill is a runtime memset, not counted."""
    return 3 if schedule == "tiled" else 2


def corner_rows(torch, w, sh, starts, value, ref, off, logits):
    """The in-level corner rows of every sample of the workload, in kernel
    order, as element offsets into the value map (int64, on the device), from
    the kernels' own cell arithmetic (msda_debug_sample_points)."""
    from scale_deformable_attention_02_b200 import msda_debug_sample_points, msda_forward_fused
    loc = torch.empty_like(off)
    msda_forward_fused(value, sh, starts, ref, off, logits, sampling_locations_out=loc)
    rows = msda_debug_sample_points(sh, starts, loc)["rows"].view(w.N, w.queries, w.M, -1)
    dev = value.device
    n = torch.arange(w.N, device=dev, dtype=torch.int64).view(-1, 1, 1, 1)
    m = torch.arange(w.M, device=dev, dtype=torch.int64).view(1, 1, -1, 1)
    elem = ((n * w.S + rows) * w.M + m) * w.D
    return elem[rows >= 0]  # row-major: item, sample, corner


def memory_floors(torch, w, offs, value, flush, reps=5):
    """Times the corner rows of this workload, in kernel order, as bare
    gathers, bare vector reductions and both (msda_debug_row_traffic): the
    floor below which no kernel's gathers and reductions can go on this GPU.
    Rows of 32 elements (D = 32: fp32 or bf16 value, fp32 gradient) only;
    else None."""
    from scale_deformable_attention_02_b200 import msda_debug_row_traffic
    if w.D != 32:
        return None
    dev = value.device
    offs = offs.to(torch.int32).contiguous()
    grad = torch.zeros(value.shape, dtype=torch.float32, device=dev)
    sink = torch.empty(16 * 256 * torch.cuda.get_device_properties(dev).multi_processor_count,
                       device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    shapes = [(dp, c * sms) for dp in (4, 8, 16) for c in (4, 8, 16)]
    out = {"rows": int(offs.numel()),
           "source": "msda_debug_row_traffic on this run's corner rows: fastest of "
                     f"{len(shapes)} (rows in flight, CTAs) launch shapes, median of {reps} "
                     "launches each after an L2 flush"}
    for mode, key in ((0, "gather_us"), (1, "reduce_us"), (2, "gather_reduce_us")):
        best = None
        for dp, ctas in shapes:
            ts = []
            for _ in range(reps + 1):
                flush.zero_()
                if mode:
                    grad.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                msda_debug_row_traffic(mode, offs, value=value if mode != 1 else None,
                                       grad=grad if mode else None, sink=sink, depth=dp,
                                       ctas=ctas)
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3)
            t = statistics.median(ts[1:])
            if best is None or t < best[0]:
                best = (t, dp, ctas)
        out[key] = best[0]
        out[key.replace("_us", "_shape")] = {"rows_in_flight": best[1], "ctas": best[2]}
    return out


def _pci_bus_id(torch, device):
    try:
        p = torch.cuda.get_device_properties(device)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


def _nvml_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    parts = [p for p in vis.split(",") if p.strip()]
    try:
        return int(parts[local])
    except Exception:
        return local


def run_e2e(args, torch, dist, world, device, stream, inp, w, st):
    """The same step through the public binding, starting from pinned host
    buffers: every step copies its inputs host -> device, runs the step's
    calls (the tile plan's sort, the forward, the backward), and copies its
    results (out and the gradients) device -> host, all inside the timed
    events.  Steps are pipelined over two device buffer sets and three streams
    (copy in, compute, copy out), so step i+1's upload and step i-1's download
    overlap step i's kernels."""
    fused = args.step == "fused"
    nbuf = 2
    queries = w.N * w.queries

    def pinned(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()

    names = ["value", "reference_points", "offsets", "logits", "grad_out"]
    h_in = {k: pinned(inp[k]) for k in names}
    res_shapes = {"out": (w.N, w.queries, w.M * w.D), "grad_value": (w.N, w.S, w.M, w.D),
                  "grad_loc": tuple(inp["offsets"].shape), "grad_attn": tuple(inp["logits"].shape)}
    if fused:
        res_shapes["grad_ref"] = tuple(inp["reference_points"].shape)
    h_out = {k: torch.empty(s, dtype=torch.float32).pin_memory() for k, s in res_shapes.items()}
    bf16 = w.value_dtype == "bf16"

    class Set:
        """One device buffer set, named as Steps names its tensors."""

    bufs = []
    for _ in range(nbuf):
        t = Set()
        t.inp = {k: torch.empty(h_in[k].shape, dtype=h_in[k].dtype, device=device)
                 for k in names}
        t.res = {k: torch.empty(s, dtype=torch.float32, device=device)
                 for k, s in res_shapes.items()}
        t.value = t.inp["value"].view(torch.bfloat16) if bf16 else t.inp["value"]
        t.ref, t.off, t.logits, t.gout = (t.inp[k] for k in names[1:])
        t.out, t.gval, t.gloc, t.gattn = (t.res[k] for k in ("out", "grad_value", "grad_loc",
                                                              "grad_attn"))
        t.gref = t.res.get("grad_ref")
        t.loc = torch.empty(tuple(inp["offsets"].shape), device=device)
        t.attn = torch.empty(tuple(inp["logits"].shape), device=device)
        if st.plan is not None:
            t.plan_buf = torch.empty_like(st.plan.buffer)
        t.loaded, t.computed, t.stored = (torch.cuda.Event() for _ in range(3))
        t.used = False
        bufs.append(t)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_comp = stream

    def step(i):
        b = bufs[i % nbuf]
        if b.used:
            s_in.wait_event(b.computed)    # step i-2 has read this input set
        with torch.cuda.stream(s_in):
            for k in names:
                b.inp[k].copy_(h_in[k], non_blocking=True)
        b.loaded.record(s_in)
        s_comp.wait_event(b.loaded)
        if b.used:
            s_comp.wait_event(b.stored)    # step i-2's results have left this set
        st.fwd(s_comp, b)
        st.bwd(s_comp, b)
        b.computed.record(s_comp)
        s_out.wait_event(b.computed)
        with torch.cuda.stream(s_out):
            for k in res_shapes:
                h_out[k].copy_(b.res[k], non_blocking=True)
        b.stored.record(s_out)
        b.used = True

    for i in range(2 * nbuf):
        step(i)
    torch.cuda.synchronize()
    n = max(1, args.e2e_steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(n):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    e1.record(s_out)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks([e0.elapsed_time(e1) / n], world, device)[0]
    h2d = sum(h_in[k].numel() * h_in[k].element_size() for k in names)
    d2h = sum(h_out[k].numel() * h_out[k].element_size() for k in res_shapes)

    # The copy floor: the same copies with no kernels, one direction at a
    # time and both at once (the pipelined step cannot beat the latter).
    def copies(do_in, do_out):
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        c0.record(s_in)
        s_out.wait_event(c0)
        for i in range(n):
            b = bufs[i % nbuf]
            if do_in:
                with torch.cuda.stream(s_in):
                    for k in names:
                        b.inp[k].copy_(h_in[k], non_blocking=True)
            if do_out:
                with torch.cuda.stream(s_out):
                    for k in res_shapes:
                        h_out[k].copy_(b.res[k], non_blocking=True)
        s_in.wait_stream(s_out)
        c1.record(s_in)
        torch.cuda.synchronize()
        return max_over_ranks([c0.elapsed_time(c1) / n], world, device)[0]

    h2d_ms, d2h_ms, both_ms = copies(True, False), copies(False, True), copies(True, True)
    floor = {"h2d_ms": h2d_ms, "d2h_ms": d2h_ms, "both_ms": both_ms,
             "h2d_GB_s": h2d / h2d_ms / 1e6, "d2h_GB_s": d2h / d2h_ms / 1e6,
             "source": "the step's own pinned copies with no kernels, same streams"}
    return {"value": queries * world / (ms / 1e3), "unit": "queries/s", "ms_per_step": ms,
            "copy_floor": floor, "frac_of_copy_floor": both_ms / ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "pipelining": f"{nbuf} device buffer sets; copy-in, compute and copy-out streams",
            "api": "scale_deformable_attention_02_b200: " + " + ".join(st.kernel_names().values())
                   + ", on pinned host buffers copied in and out every step"}


# ---------------------------------------------------------------------------
# CPU oracle legs (the oracle is test infrastructure; only these legs run it)
# ---------------------------------------------------------------------------
def _oracle_sample(w, inp, frac_queries: int):
    """Every frac-th query of every batch entry (the oracle's cost per query
    is uniform, so a strided sample keeps the workload's mix)."""
    qs = np.arange(0, w.queries, frac_queries)
    pick = lambda a: np.ascontiguousarray(a[:, qs])  # noqa: E731
    return {"value": inp["value"], "spatial_shapes": inp["spatial_shapes"],
            "reference_points": pick(inp["reference_points"]), "offsets": pick(inp["offsets"]),
            "logits": pick(inp["logits"]), "grad_out": pick(inp["grad_out"]),
            "queries": w.N * len(qs)}


def _oracle_step(oracle, s):
    out, loc, A = oracle.forward_fused(s["value"], s["spatial_shapes"], s["reference_points"],
                                       s["offsets"], s["logits"])
    oracle.backward(s["value"], s["spatial_shapes"], loc, A, s["grad_out"])


def cpu_baseline(w, inp, min_seconds: float = 10.0):
    import oracle
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    s = _oracle_sample(w, inp, 1)
    t0 = time.perf_counter()
    passes = 0
    while True:
        _oracle_step(oracle, s)
        passes += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or passes >= 20:
            break
    # one thread, on every 16th query
    oracle.set_threads(1)
    s1 = _oracle_sample(w, inp, 16)
    t1 = time.perf_counter()
    _oracle_step(oracle, s1)
    el1 = time.perf_counter() - t1
    oracle.set_threads(threads)
    return {"value": s["queries"] * passes / el, "unit": "queries/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{passes} full pass(es) of the workload ({s['queries']} queries each: "
                      f"fused forward + backward) on the plain C oracle, fp64 accumulation, "
                      f"OpenMP over {threads} threads, {el:.1f} s",
            "single_thread": {"value": s1["queries"] / el1, "unit": "queries/s", "cores": 1,
                              "sample": f"every 16th query ({s1['queries']} queries), one pass, "
                                        f"{el1:.1f} s"}}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    import oracle
    w = rank_workload(args.workload, 0)
    inp = wl.make_inputs(w)
    stride = 8 if args.workload == "stress" else 4
    s = _oracle_sample(w, inp, stride)
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    for _ in range(args.warmup):
        _oracle_step(oracle, s)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_step(oracle, s)
        times.append(time.perf_counter() - t0)
    sec = statistics.fmean(times)
    qps = s["queries"] / sec
    sample = (f"every {stride}th query of each of the {w.N} batch entries ({s['queries']} "
              f"queries per step), fused forward + backward on the plain C oracle")
    line = {
        "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy PCG64)",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "value_dtype": w.value_dtype,
                   "global_batch": w.N, "parallelism": "host cores (OpenMP)"},
        "impl": "reference",
        "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
