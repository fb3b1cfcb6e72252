#!/usr/bin/env python
"""Benchmark of the selective-scan forward on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

For N > 1 launch one rank per GPU with torch.distributed.run; each rank runs the
same shape on its own shard of the job (batch rows are independent, so there is
no data-path collective: weak scaling), the timed region is bracketed by a
barrier and a device synchronise, and the slowest rank's time is reported.

A step is one full forward over the workload (discretise, recurrence, readout,
final state) with inputs already resident in HBM.  Rank 0 prints one JSON line.
``--impl reference`` times the fp64 CPU oracle instead (host cores, rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_32_b200 import workloads as W  # noqa: E402

METRIC = "selective-scan elements (B*L*D)/s"
UNIT = "elements/s"
L2_BYTES = 126 * 1024 * 1024
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
SM_COUNT = 148
SM_MAX_MHZ = 1965.0
# ALU roofline of one state update on B200 (per SM per clock): 16 MUFU ex2 and
# 128 FP32 FMA-pipe lanes.  An update needs one 2^x and four FMA-pipe ops
# (delta*A, B*(delta*u), Abar*h + Bbar u, y += C*h); a 2^x can instead be
# computed on the FMA pipe with eight ops (range reduction + degree-5
# polynomial).  With a fraction f of the exponents in software the MUFU pipe
# allows 16 / (1 - f) updates per clock and the FMA pipe 128 / (4 + 8 f); the
# two are equal at f = 1/4, i.e. 16 / (3/4) = 21.33 updates per SM per clock.
ALU_UPDATES_PER_SM_CLK = 16.0 / (1.0 - 0.25)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("sm_max_mhz", SM_MAX_MHZ)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, SM_MAX_MHZ, "fallback"


def strip_comments(src: str) -> str:
    """C/C++/CUDA source without comments and blank lines (string literals in these
    sources hold no comment markers), so that a comment edit keeps the hash."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


SSD_SOURCES = ("kernel_ssd.cuh", "ssd.cu")
HOST_ONLY_SOURCES = ("host_pipe.cu",)  # copies and sub-plan calls: no kernel launch of its own


def kernel_sources_hash(read=None, family: str = "scan") -> str:
    """sha256 over the code (comments stripped) of one family of forward kernels and
    their host code, to tell whether a stored ncu figure is current: "scan" (the
    selective-scan kernels: every CUDA source but the backward's and the SSD form's)
    or "ssd" (the SSD form's sources and the shared device utilities); the host-buffer
    pipeline's file launches nothing itself and is in neither.  ``read(name)`` returns a
    file's text (default: the working tree)."""
    import hashlib
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "selective_state_space_32_b200", "csrc")
    names = [n for n in sorted(os.listdir(cdir))
             if n.endswith((".cu", ".cuh")) and "backward" not in n and n not in HOST_ONLY_SOURCES]
    if family == "ssd":
        names = [n for n in names if n in SSD_SOURCES or n == "device_utils.cuh"]
    else:
        names = [n for n in names if n not in SSD_SOURCES]
    for name in names:
        if read is None:
            with open(os.path.join(cdir, name), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(name)
        h.update(name.encode() + b"\0" + strip_comments(text).encode())
    return h.hexdigest()


def measured_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the dominant kernel from the committed
    ncu capture (profiles/traffic.json), or None if absent or taken on other sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        family = "ssd" if workload in W.SSD_WORKLOADS else "scan"
        if t.get("kernel_sources_sha256", {}).get(family) != kernel_sources_hash(family=family):
            return None
        v = t["workloads"][workload]["dram_bytes_per_launch"]
        return float(v)
    except Exception:
        return None


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.001):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------- CPU oracle --

def cpu_oracle_rate(g, w, min_seconds=10.0, max_seconds=30.0):
    """Time the fp64 oracle as it stands on this host's cores: full passes over the
    workload until at least ``min_seconds`` elapsed.  Returns (elements/s, cores, sample)."""
    from oracle import oracle as O
    v = _oracle_values(g, w)
    cores = O.host_threads()
    n, t0 = 0, time.perf_counter()
    while True:
        O.forward(v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], w.zoh, nthreads=cores,
                  delta_bias=v["delta_bias"], softplus=w.fused, z=v["z"])
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or el + el / n > max_seconds:
            break
    return n * w.elements / el, cores, f"{n} full pass(es) over the workload ({w.elements} elements each) in {el:.2f} s"


def workload_config(w, world: int) -> dict:
    """The ``config`` object of a JSON line: the same keys for both arms, so a line of
    ours and a reference line of the same workload compare as the same configuration."""
    alg_bytes = w.algorithmic_bytes()
    return {"workload": f"{w.name}: B={w.B} L={w.L} D={w.D} N={w.N} io={w.dtype} "
                        f"{'ZOH' if w.zoh else 'Euler'} h0={'yes' if w.h0_std else 'no'}"
                        f"{' resets=' + str(w.reset_frac) if w.reset_frac else ''}"
                        f"{' fused softplus(delta+bias), y*silu(z)' if w.fused else ''}",
            "B": w.B, "L": w.L, "D": w.D, "N": w.N, "io_dtype": w.dtype,
            "parallelism": f"dp{world} (independent batch-row shards, no collective)",
            "l2": (f"inputs larger than L2 ({alg_bytes / 1e6:.0f} MB per step vs "
                   f"{L2_BYTES / 2**20:.0f} MiB L2); no flush" if alg_bytes >= L2_BYTES else
                   f"working set below L2 ({alg_bytes / 1e6:.0f} MB vs {L2_BYTES / 2**20:.0f} MiB): "
                   f"{rotating_sets(w)} input/state sets ({rotating_sets(w) * alg_bytes / 1e6:.0f} MB) "
                   f"used in turn, one per step (as the layers of a model), steps back to back; no flush")}


def graph_of_steps(step, count: int, stream, dev):
    """A CUDA graph of ``count`` calls ``step(i, s)`` captured on a side stream, for steps
    of a few microseconds whose Python launch cost would otherwise set the pace; None if
    the capture fails.  Only for schedules without launch epochs (decode, step)."""
    import torch
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(count):
                step(i, side)
        stream.wait_stream(side)
        return g
    except Exception:
        return None


def rotating_sets(w) -> int:
    """Distinct input/state sets a workload whose working set fits in L2 is timed over
    (one per step, in turn), so that together they exceed L2 three times over."""
    alg = w.algorithmic_bytes()
    return 1 if alg >= L2_BYTES else -(-3 * L2_BYTES // alg)


# ------------------------------------------------------- multi-rank logic --

def shard_seed(w, rank: int) -> int:
    """Seed of rank r's shard: batch rows [r*B, (r+1)*B) of an N*B-row job."""
    return W.SEED_BASE + w.index + 1000 * rank


def max_over_ranks(values, world: int, device=None):
    """Element-wise maximum of a list of floats over all ranks (timings)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# -------------------------------------------------------------- our arm --

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from selective_state_space_32_b200 import sscan as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[args.workload]
    # shard: rank r owns batch rows [r*B, (r+1)*B) of an N*B-row job (own seed)
    g = W.generate(w.B, w.L, w.D, w.N, w.dtype, w.h0_std, w.reset_frac,
                   seed=shard_seed(w, rank), fused=w.fused)
    tdt = torch.float32 if w.dtype == "f32" else torch.bfloat16

    def host(x, dt):
        if x is None:
            return None
        if dt == "bf16":
            t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        return t.pin_memory()

    hin = {"u": host(g["u"], w.dtype), "delta": host(g["delta"], w.dtype),
           "A": host(g["A"], "f32"), "B": host(g["B"], w.dtype), "C": host(g["C"], w.dtype),
           "h0": host(g["h0"], "f32"), "delta_bias": host(g["delta_bias"], "f32"),
           "z": host(g["z"], w.dtype)}
    din = {k: (None if v is None else v.to(dev)) for k, v in hin.items()}
    plan = S.Plan(w.B, w.L, w.D, w.N, tdt, w.zoh, delta_softplus=w.fused)
    ws = plan.new_workspace(dev)
    y = torch.empty((w.B, w.L, w.D), dtype=tdt, device=dev)
    hf = torch.empty((w.B, w.D, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # a working set below L2 is timed over several input/state sets in turn (no L2 reuse)
    nsets = rotating_sets(w)
    sets = [(din, y, hf)] + [({k: (None if v is None else v.clone()) for k, v in din.items()},
                              torch.empty_like(y), torch.empty_like(hf)) for _ in range(nsets - 1)]

    def step(i=0, st=None):
        d, yy, hh = sets[i % nsets]
        plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"],
                     y=yy, h_final=hh, workspace=ws, stream=st or stream,
                     delta_bias=d["delta_bias"], z=d["z"])

    for i in range(max(args.warmup, nsets)):
        step(i)
    torch.cuda.synchronize(dev)
    if plan.status(stream) != S.OK:
        raise RuntimeError("device status word reported an error during warm-up")
    # steps of a few microseconds (rotated sets; no launch epochs) replay as one CUDA graph
    graph = (graph_of_steps(step, args.steps, stream, dev)
             if nsets > 1 and plan.describe().startswith(("kernel=decode", "kernel=step")) else None)
    if graph is not None:
        with torch.cuda.stream(stream):
            graph.replay()  # a warm-up replay
        torch.cuda.synchronize(dev)

    # ---- timed region: K steps, events around every launch (kernel time) ----
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        if graph is not None:
            with torch.cuda.stream(stream):
                graph.replay()
        else:
            for i in range(args.steps):
                if nsets == 1:  # a step of a few microseconds (rotated sets) is not split by events
                    ev[i][0].record(stream)
                step(i)
                if nsets == 1:
                    ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    kern_ms = [a.elapsed_time(b) for a, b in ev] if nsets == 1 else [elapsed_ms / args.steps] * args.steps
    launch_mode = ("one CUDA graph of the K steps" if graph is not None else
                   "direct launches, back to back" if nsets > 1 else "direct launches, events around each")
    if plan.status(stream) != S.OK:
        raise RuntimeError("device status word reported an error in the timed region")

    # ---- end to end: host buffers through the public API, copies inside ----
    out_h = (torch.empty(y.shape, dtype=y.dtype).pin_memory(),
             torch.empty(hf.shape, dtype=hf.dtype).pin_memory())
    e2e_steps = max(1, min(args.steps, 20))

    def e2e_step():
        S.forward_host(hin["u"], hin["delta"], hin["A"], hin["B"], hin["C"], hin["h0"],
                       zoh=w.zoh, device=dev, out=out_h, delta_bias=hin["delta_bias"],
                       delta_softplus=w.fused, z=hin["z"], stream=stream)

    for _ in range(min(args.warmup, 3)):
        e2e_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    h2d = sum(v.numel() * v.element_size() for v in hin.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in out_h)

    # ---- max over ranks ----
    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], world, dev)

    if rank != 0:
        return None
    hbm_peak, sm_max, peak_src = load_peaks()
    kmean = sum(kern_ms) / len(kern_ms)
    value = w.elements * args.steps * world / (elapsed_ms / 1e3)
    alg_bytes = w.algorithmic_bytes()
    hbm_achieved = alg_bytes / (kmean / 1e3) / 1e9
    upd_rate = w.updates / (kmean / 1e3) / 1e9
    alu_peak = ALU_UPDATES_PER_SM_CLK * SM_COUNT * sm_max * 1e6 / 1e9
    mufu_peak = 16.0 * SM_COUNT * sm_max * 1e6 / 1e9     # one exp2 per update, MUFU only
    kernel_name = "sscan_" + plan.describe().split()[0].split("=")[1] + "_kernel"
    traffic = measured_traffic(args.workload)
    cpu_value, cores, sample = cpu_oracle_rate(g, w, args.cpu_seconds, 3 * args.cpu_seconds)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, world),
        "timing": launch_mode,
        "roofline": ({"bound": "alu", "achieved": upd_rate, "peak": alu_peak,
                      "unit": "Gupdates/s", "frac": upd_rate / alu_peak, "traffic": traffic,
                      "kernel": kernel_name, "schedule": plan.describe(),
                      "peak_basis": f"{ALU_UPDATES_PER_SM_CLK:.1f} state updates/SM/clk "
                                    f"(16 MUFU + 128 FMA lanes) x {SM_COUNT} SMs x {sm_max:.0f} MHz",
                      "mufu_only_peak": mufu_peak, "mufu_only_frac": upd_rate / mufu_peak}
                     if w.L > 1 else
                     # one token: a stream over the state, bound by HBM
                     {"bound": "hbm", "achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s",
                      "frac": hbm_achieved / hbm_peak, "traffic": traffic, "kernel": kernel_name,
                      "schedule": plan.describe(), "peak_basis": f"{peak_src} copy bandwidth"}),
        "hbm": {"achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": hbm_achieved / hbm_peak, "peak_source": peak_src,
                "algorithmic_bytes_per_step": alg_bytes},
        "kernel_ms": {"mean": kmean, "min": min(kern_ms), "max": max(kern_ms)},
        "e2e": {"value": w.elements * e2e_steps * world / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": {"value": cpu_value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
    }
    if args.per_config:
        others = [n for n in W.ORDER[1:] + ["mamba130m_fused_f32", "mamba1p4b_fused_bf16", "decode_b256_f32"]
                  if n != args.workload]
        out["per_config"] = time_other_configs(others, dev, stream, sm_max, hbm_peak)
        for name, sw in W.SSD_WORKLOADS.items():
            if name == "ssd_small":
                continue
            try:
                _, sd = ssd_to_device(W.make_ssd_inputs(sw), dev)
                ms = time_ssd(sw, sd, dev, stream, 20, 3)
                km = sum(ms) / len(ms)
                out["per_config"][name] = {"kernel_ms": km, "elements_per_s": sw.elements / (km / 1e3),
                                           **ssd_roofline(sw, km, hbm_peak, read_peaks())}
                del sd
            except Exception as e:
                out["per_config"][name] = {"error": str(e)[:200]}
    if args.per_config:
        out["backward"] = time_backward(dev, stream)
    plan.close()
    return out


def to_device(g, dev):
    """Generated arrays -> CUDA tensors in their storage dtype (bf16 bit patterns -> bfloat16)."""
    import torch

    def t(x, dt):
        if x is None:
            return None
        if dt == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)
    dt = g["dtype"]
    return {"u": t(g["u"], dt), "delta": t(g["delta"], dt), "A": t(g["A"], "f32"), "B": t(g["B"], dt),
            "C": t(g["C"], dt), "h0": t(g["h0"], "f32"), "delta_bias": t(g.get("delta_bias"), "f32"),
            "z": t(g.get("z"), dt)}


def time_other_configs(names, dev, stream, sm_max, hbm_peak, launches: int = 20, warmup: int = 3):
    """Kernel time of each named workload in this run (CUDA events around each launch on
    the launching stream, inputs resident in HBM), with its element rate and its HBM and
    ALU roofline fractions.  A figure per configuration beside the headline line."""
    import torch
    from selective_state_space_32_b200 import sscan as S
    out = {}
    alu_peak = ALU_UPDATES_PER_SM_CLK * SM_COUNT * sm_max * 1e6 / 1e9
    for name in names:
        w = W.WORKLOADS[name]
        try:
            d = to_device(W.make_inputs(w), dev)
            tdt = torch.float32 if w.dtype == "f32" else torch.bfloat16
            plan = S.Plan(w.B, w.L, w.D, w.N, tdt, w.zoh, delta_softplus=w.fused)
            ws = plan.new_workspace(dev)
            y = torch.empty((w.B, w.L, w.D), dtype=tdt, device=dev)
            hf = torch.empty((w.B, w.D, w.N), dtype=torch.float32, device=dev)
            # a working set that fits in L2 is timed over several input/state sets in turn
            nsets = rotating_sets(w)
            sets = [(d, y, hf)] + [({k: (None if v is None else v.clone()) for k, v in d.items()},
                                    torch.empty_like(y), torch.empty_like(hf)) for _ in range(nsets - 1)]

            def step(i=0, st=None):
                dd, yy, hh = sets[i % nsets]
                plan.forward(dd["u"], dd["delta"], dd["A"], dd["B"], dd["C"], dd["h0"], y=yy, h_final=hh,
                             workspace=ws, stream=st or stream, delta_bias=dd["delta_bias"], z=dd["z"])
            for i in range(max(warmup, nsets)):
                step(i)
            graph = (graph_of_steps(step, launches, stream, dev)
                     if nsets > 1 and plan.describe().startswith(("kernel=decode", "kernel=step")) else None)
            if graph is not None:
                with torch.cuda.stream(stream):
                    graph.replay()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(launches if nsets == 1 else 1)]
            torch.cuda.synchronize(dev)
            if nsets == 1:  # events around every launch
                for i, (a, b) in enumerate(ev):
                    a.record(stream)
                    step(i)
                    b.record(stream)
            else:  # steps of a few microseconds: back to back (one CUDA graph), one pair of events
                ev[0][0].record(stream)
                if graph is not None:
                    with torch.cuda.stream(stream):
                        graph.replay()
                else:
                    for i in range(launches):
                        step(i)
                ev[0][1].record(stream)
            torch.cuda.synchronize(dev)
            if plan.status(stream) != S.OK:
                raise RuntimeError("device status word reported an error")
            ms = sum(a.elapsed_time(b) for a, b in ev) / launches
            gbs = w.algorithmic_bytes() / (ms / 1e3) / 1e9
            upd = w.updates / (ms / 1e3) / 1e9
            out[name] = {"kernel_ms": ms, "elements_per_s": w.elements / (ms / 1e3),
                         "hbm_gbs": gbs, "hbm_frac": gbs / hbm_peak, "alu_frac": upd / alu_peak,
                         "mufu_only_frac": upd / (16.0 * SM_COUNT * sm_max * 1e6 / 1e9),
                         "launches": launches, "schedule": plan.describe(),
                         "l2": (f"{nsets} input/state sets used in turn (working set below L2)" if nsets > 1
                                else "inputs larger than L2; no flush"),
                         "launch": ("one CUDA graph of the launches" if graph is not None else
                                    "direct launches" if nsets > 1 else "direct launches, events around each")}
            plan.close()
            del d, y, hf, ws, sets, graph
            torch.cuda.empty_cache()
        except Exception as e:  # reported, never fatal for the headline line
            out[name] = {"error": str(e)[:200]}
    return out


def time_backward(dev, stream, name: str = "mamba130m_f32", reps: int = 5):
    """The backward pass (sscan_backward) on the named workload's inputs (a fixed
    shape, whatever the headline workload is), dy = 1: mean of ``reps`` launches
    (CUDA events), reported beside the forward."""
    import torch
    from selective_state_space_32_b200 import sscan as S
    try:
        w = W.WORKLOADS[name]
        din = to_device(W.make_inputs(w), dev)
        tdt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        plan = S.Plan(w.B, w.L, w.D, w.N, tdt, w.zoh)
        dy = torch.ones((w.B, w.L, w.D), dtype=tdt, device=dev)
        f = lambda: plan.backward(din["u"], din["delta"], din["A"], din["B"], din["C"], din["h0"], dy,
                                  stream=stream)
        f()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            f()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b) / reps
        plan.close()
        return {"workload": name, "kernel_ms": ms, "value": w.elements / (ms / 1e3), "unit": UNIT,
                "launches": reps, "note": "sscan_backward (du, ddelta, dA, dB, dC, dh0), dy = 1; "
                "3 exponentials per state update (forward checkpoints, recompute, reverse)",
                "mufu_only_frac": 3 * w.updates / (ms / 1e3) / (16.0 * SM_COUNT * SM_MAX_MHZ * 1e6)}
    except Exception as e:  # reported, never fatal for the forward line
        return {"error": str(e)[:200]}


# ------------------------------------------------------------- SSD arm --

def ssd_config(w, world: int) -> dict:
    """``config`` of an SSD line (the same keys for both arms)."""
    alg = w.algorithmic_bytes()
    return {"workload": f"{w.name}: Mamba-2 SSD B={w.B} L={w.L} H={w.H} P={w.P} N={w.N} io=bf16 "
                        f"(delta fp32) h0={'yes' if w.h0_std else 'no'}",
            "B": w.B, "L": w.L, "H": w.H, "P": w.P, "N": w.N, "io_dtype": "bf16",
            "parallelism": f"dp{world} (independent batch-row shards, no collective)",
            "l2": f"inputs larger than L2 ({alg / 1e6:.0f} MB per step vs {L2_BYTES / 2**20:.0f} MiB L2); no flush"}


def ssd_to_device(g, dev):
    import torch
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    f32 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32))
    host = {"x": bf(g["x"]), "delta": f32(g["delta"]), "A": f32(g["A"]), "B": bf(g["B"]), "C": bf(g["C"]),
            "h0": f32(g["h0"])}
    return host, {k: (None if v is None else v.to(dev)) for k, v in host.items()}


def ssd_oracle_values(g):
    w = lambda a: W.bf16_bits_to_f32(a).astype(np.float64)
    return (w(g["x"]), g["delta"].astype(np.float64), g["A"].astype(np.float64), w(g["B"]), w(g["C"]),
            None if g["h0"] is None else g["h0"].astype(np.float64))


def ssd_oracle_rate(g, w, pairs: int):
    """The fp64 SSD oracle (block-chunked form, pinned to the quadratic form) as it stands,
    single-threaded, on ``pairs`` (batch row, head) sequences of the workload (each is an
    independent problem).  Returns (elements/s, sample description)."""
    from oracle import ssd_oracle as O
    x, dl, A, Bm, Cm, h0 = ssd_oracle_values(g)
    sel = [(i % w.B, (7 * i) % w.H) for i in range(pairs)]
    subs = [(np.ascontiguousarray(x[b:b + 1, :, h:h + 1]), np.ascontiguousarray(dl[b:b + 1, :, h:h + 1]),
             A[h:h + 1], np.ascontiguousarray(Bm[b:b + 1]), np.ascontiguousarray(Cm[b:b + 1]),
             None if h0 is None else np.ascontiguousarray(h0[b:b + 1, h:h + 1])) for b, h in sel]
    t0 = time.perf_counter()
    for sub in subs:
        O.ssd_forward_chunked(*sub, block=64)
    el = time.perf_counter() - t0
    return pairs * w.L * w.P / el, f"{pairs} of {w.B * w.H} (batch row, head) sequences, one core, {el:.2f} s"


def time_ssd(w, d, dev, stream, launches: int, warmup: int, status=None):
    """Mean kernel time (ms) of sscan_ssd_forward over ``launches`` launches, CUDA events on
    the launching stream around each launch, inputs resident in HBM."""
    import torch
    from selective_state_space_32_b200 import sscan as S
    y = torch.empty((w.B, w.L, w.H, w.P), dtype=torch.bfloat16, device=dev)
    hf = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device=dev)
    step = lambda: S.ssd_forward(d["x"], d["delta"], d["A"], d["B"], d["C"], d["h0"], y=y, h_final=hf,
                                 status=status, stream=stream)
    for _ in range(warmup):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return [a.elapsed_time(b) for a, b in ev]


def ssd_roofline(w, kms, hbm_peak, peaks):
    gbs = w.algorithmic_bytes() / (kms / 1e3) / 1e9
    tfl = w.flops() / (kms / 1e3) / 1e12
    bf16 = peaks.get("bf16_tflops", 1590.0)
    return {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
            "traffic": measured_traffic(w.name),
            "kernel": "ssd_forward_kernel", "tensor": {"achieved_tflops": tfl, "peak_tflops": bf16,
                                                       "frac": tfl / bf16,
                                                       "flops_per_step": w.flops()}}


def run_ours_ssd(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from selective_state_space_32_b200 import sscan as S
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = W.SSD_WORKLOADS[args.workload]
    g = W.generate_ssd(w.B, w.L, w.H, w.P, w.N, w.h0_std, seed=W.SEED_BASE + w.index + 1000 * rank)
    hin, din = ssd_to_device(g, dev)
    hin = {k: (None if v is None else v.pin_memory()) for k, v in hin.items()}
    stream = torch.cuda.current_stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y = torch.empty((w.B, w.L, w.H, w.P), dtype=torch.bfloat16, device=dev)
    hf = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device=dev)
    step = lambda: S.ssd_forward(din["x"], din["delta"], din["A"], din["B"], din["C"], din["h0"], y=y, h_final=hf,
                                 status=status, stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    if int(status.item()) != 0:
        raise RuntimeError("SSD kernel reported a wait that gave up")
    # end to end: pinned host buffers, copies in and out inside the timed region
    out_h = (torch.empty(y.shape, dtype=y.dtype).pin_memory(), torch.empty(hf.shape, dtype=hf.dtype).pin_memory())
    e2e_steps = max(1, min(args.steps, 20))

    def e2e_step():
        dv = {k: (None if v is None else v.to(dev, non_blocking=True)) for k, v in hin.items()}
        yy, hh = S.ssd_forward(dv["x"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["h0"], stream=stream)
        out_h[0].copy_(yy, non_blocking=True)
        out_h[1].copy_(hh, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()

    for _ in range(min(args.warmup, 3)):
        e2e_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], world, dev)
    if rank != 0:
        return None
    hbm_peak, sm_max, peak_src = load_peaks()
    kmean = sum(kern_ms) / len(kern_ms)
    cpu_value, sample = ssd_oracle_rate(g, w, args.ssd_oracle_pairs)
    h2d = sum(v.numel() * v.element_size() for v in hin.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in out_h)
    return {
        "metric": METRIC, "value": w.elements * args.steps * world / (elapsed_ms / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (fp32 accumulate)",
        "data": "synthetic", "config": ssd_config(w, world),
        "roofline": ssd_roofline(w, kmean, hbm_peak, read_peaks()),
        "kernel_ms": {"mean": kmean, "min": min(kern_ms), "max": max(kern_ms)},
        "e2e": {"value": w.elements * e2e_steps * world / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": args.steps, "clocks": clk.summary(),
        "cpu_baseline": {"value": cpu_value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
    }


def run_reference_ssd(args):
    w = W.SSD_WORKLOADS[args.workload]
    g = W.make_ssd_inputs(w)
    pairs = max(1, args.ssd_oracle_pairs)
    for _ in range(args.warmup):
        ssd_oracle_rate(g, w, 1)
    rates = [ssd_oracle_rate(g, w, pairs)[0] for _ in range(args.steps)]
    value = len(rates) / sum(1.0 / r for r in rates)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * pairs * w.L * w.P / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": ssd_config(w, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{pairs} (batch row, head) sequences per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def read_peaks() -> dict:
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f)
    except Exception:
        return {}


# -------------------------------------------------------- reference arm --

def _oracle_values(g, w):
    """The workload's inputs as the fp64 values the oracle reads (bf16 widened exactly)."""
    v = {k: (None if g.get(k) is None else W.as_f32(g[k], g["dtype"]).astype(np.float64))
         for k in ("u", "delta", "B", "C", "z")}
    v["A"] = g["A"].astype(np.float64)
    v["h0"] = None if g["h0"] is None else g["h0"].astype(np.float64)
    v["delta_bias"] = None if g.get("delta_bias") is None else g["delta_bias"].astype(np.float64)
    return v


def _sub_problem(v, nb: int, nd: int) -> dict:
    """Batch rows [0, nb) and channels [0, nd) of the workload as contiguous arrays (rows
    are independent, so this is an exact sub-problem of the same workload)."""
    cut = lambda x: None if x is None else np.ascontiguousarray(x[:nb, :, :nd])
    return {"u": cut(v["u"]), "delta": cut(v["delta"]), "z": cut(v["z"]),
            "B": np.ascontiguousarray(v["B"][:nb]), "C": np.ascontiguousarray(v["C"][:nb]),
            "A": np.ascontiguousarray(v["A"][:nd]),
            "h0": None if v["h0"] is None else np.ascontiguousarray(v["h0"][:nb, :nd]),
            "delta_bias": None if v["delta_bias"] is None else np.ascontiguousarray(v["delta_bias"][:nd])}


def run_reference(args):
    """The reference arm: the fp64 oracle (the only reference: the pages ship no runnable
    code) on the host cores, as it stands.  Every step is one ``O.forward`` over the same
    contiguous sub-problem of the workload (leading batch rows and channels, prepared
    before the timed region), sized so that warm-up and timed steps together take about
    ``--ref-seconds``; the value is the sub-problem's elements per second."""
    w = W.WORKLOADS[args.workload]
    g = W.make_inputs(w)
    from oracle import oracle as O
    v = _oracle_values(g, w)
    cores = O.host_threads()
    run = lambda p: O.forward(p["u"], p["delta"], p["A"], p["B"], p["C"], p["h0"], w.zoh,
                              nthreads=cores, delta_bias=p["delta_bias"], softplus=w.fused, z=p["z"])
    # probe: one batch row, a slice of channels, to size the step
    nd0 = max(1, min(w.D, 2 * cores))
    probe = _sub_problem(v, 1, nd0)
    t0 = time.perf_counter()
    run(probe)
    per_elem = (time.perf_counter() - t0) / (w.L * nd0)
    per_step = max(0.05, args.ref_seconds / (args.steps + args.warmup))
    want = max(1, int(per_step / max(per_elem, 1e-12) / w.L))  # (b, d) rows per step
    nb = max(1, min(w.B, want // w.D))
    nd = w.D if nb > 1 else max(1, min(w.D, want))
    sub = _sub_problem(v, nb, nd)
    for _ in range(args.warmup):
        run(sub)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run(sub)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    elems = nb * w.L * nd
    value = elems * args.steps / tot
    sample = (f"batch rows [0, {nb}) x channels [0, {nd}) of the workload ({elems} of {w.elements} "
              f"elements) per step, one oracle call each")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(w, int(os.environ.get("WORLD_SIZE", "1"))),  # our arm's config at this N
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="longseq_bf16", choices=sorted(W.WORKLOADS) + sorted(W.SSD_WORKLOADS))
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch rows (small cases for profiling); 0 keeps it")
    ap.add_argument("--length", type=int, default=0,
                    help="override the workload's sequence length (small cases for profiling); 0 keeps it")
    ap.add_argument("--ssd-oracle-pairs", type=int, default=4,
                    help="(batch row, head) sequences the SSD oracle baseline times")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--per-config", type=int, default=1,
                    help="also time the kernel on the other configurations (rank 0, outside the timed region)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="minimum host time spent timing the CPU oracle baseline")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="host time of the reference (oracle) arm's warm-up and timed steps together")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus > 1 needs one process per GPU (torch.distributed.run)")
    if args.batch > 0 or args.length > 0:
        import dataclasses
        table = W.SSD_WORKLOADS if args.workload in W.SSD_WORKLOADS else W.WORKLOADS
        w0 = table[args.workload]
        table[args.workload] = dataclasses.replace(w0, B=args.batch or w0.B, L=args.length or w0.L)
    is_ssd = args.workload in W.SSD_WORKLOADS
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference_ssd(args) if is_ssd else run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = (run_ours_ssd if is_ssd else run_ours)(args, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
