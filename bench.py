#!/usr/bin/env python
"""Throughput of exact tiled attention (forward + backward) on B200, one JSON line.

A step is one pass of the whole path over one batch: fa_fwd (O, lse) then fa_bwd (dQ, dK, dV)
on the long-context causal workload (B1 H16 N16384 d128, Q,K ~ 2 N(0,1), bf16), inputs
resident in HBM.  FLOPs count only unmasked (i, j) pairs P: 4 d P forward, 10 d P backward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) every rank runs its own replica of the workload (the (b, h) problems
are independent, so there is no data-path collective; scaling is weak) and the time is the
max over ranks.  ``--impl reference`` times the FP64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

WORKLOAD = "long_causal"
METRIC = "attention fwd/bwd TFLOP/s on 1 B200 and % of BF16 tensor peak; max err vs FP64"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(syn.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="time fa_bwd_deterministic (dQ without atomics) as the step's backward")
    ap.add_argument("--cpu-rows", type=int, default=16384,
                    help="query rows in the oracle's timed sample")
    ap.add_argument("--ref-rows", type=int, default=1024,
                    help="query rows per step of the reference (oracle) arm")
    return ap.parse_args()


# ----------------------------------------------------------------------------- accounting
def flops(x: dict, H: int) -> tuple[float, float]:
    kv = None if x["kv_len"] is None else x["kv_len"].numpy()
    bm = None if x["block_mask"] is None else x["block_mask"].numpy()
    P = float(syn.allowed_pairs(x["N"], x["causal"], kv, x["B"], bm).sum()) * H
    return 4.0 * x["d"] * P, 10.0 * x["d"] * P


def row_pairs(x: dict, rows: np.ndarray) -> np.ndarray:
    """Unmasked keys of each flat row (counting only; used for the oracle sample's FLOPs)."""
    N, H = x["N"], x["q"].shape[1]
    i = rows % N
    b = rows // N // H
    L = np.full(len(rows), N) if x["kv_len"] is None else x["kv_len"].numpy()[b]
    n = np.minimum(i + 1, L) if x["causal"] else L.copy()
    if x["block_mask"] is not None:
        bm = x["block_mask"].numpy()
        n = np.array([sum(max(0, min((J + 1) * 128, Lr, (ir + 1) if x["causal"] else Lr) - J * 128)
                          for J in range(bm.shape[1]) if bm[ir // 128, J])
                      for ir, Lr in zip(i, L)])
    return n.astype(np.float64)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def select_peak(peaks: dict, clocks: dict) -> tuple[float, str]:
    """The bf16 roof for a kernel timed in this run.  The burst figure (cuBLAS bf16 in a short
    burst at the maximum SM clock) applies when the timed region's median SM clock under load
    is at its maximum, as in a short region; the sustained figure (the same GEMM settled under
    the power cap, at a lower clock) only when the region's clock settled below the maximum.
    Without a clock record the burst figure is used, the larger of the two."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    sm = clocks.get("sm_mhz")
    smax = clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    if sm is None or smax is None:
        return burst, "bf16_tflops (burst): no clock record, the larger roof"
    if float(sm) >= 0.97 * float(smax):
        return burst, (f"bf16_tflops (burst): median SM clock under load {sm:.0f} MHz is at its "
                       f"maximum {smax:.0f} MHz")
    return sustained, (f"bf16_tflops_sustained: median SM clock under load {sm:.0f} MHz settled "
                       f"below its maximum {smax:.0f} MHz")


def csrc_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "exact_io_aware_98_b200", "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel, {}).get(workload, {})
    if e.get("csrc_hash") != csrc_hash():
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.ok = False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # no NVML: report the absence, never guess
            self.err = repr(exc)
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if bits & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        self._stop.set()
        self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- ranks
def init_distributed(backend: str, timeout_s: int = 120):
    """One process per GPU (torchrun env); returns torch.distributed or None when WORLD_SIZE=1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return None
    import torch.distributed as tdist
    tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return tdist


def max_over_ranks(values, dist, device) -> list:
    """Element-wise max over ranks of per-rank timings (the job is as slow as its slowest rank)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# MUFU (special-function unit) throughput for ex2: 16 results per clock per SM, measured on a
# B200 with independent ex2.approx chains on every SM (the packed f16x2 form gives the same 16);
# 148 SMs on a B200.
MUFU_PER_CLK_PER_SM = 16
N_SM = 148


def step_stats(ms: list) -> dict:
    """Median and p10/p90 of per-step durations (the mean is reported beside them)."""
    if len(ms) < 2:
        return {"median_ms": round(ms[0], 4)} if ms else {}
    q = statistics.quantiles(ms, n=10, method="inclusive")
    return {"median_ms": round(statistics.median(ms), 4), "p10_ms": round(q[0], 4),
            "p90_ms": round(q[-1], 4)}


def exp_roof(pairs: float, ms: float, sm_mhz) -> dict:
    """The second roof of both passes: one exponential per unmasked (query, key) pair, against
    the MUFU ex2 rate at the sampled SM clock.  The forward takes part of its exponentials on
    the FMA pipe, so its fraction can read above what MUFU alone could deliver."""
    mhz = float(sm_mhz) if sm_mhz else 1965.0
    peak = MUFU_PER_CLK_PER_SM * N_SM * mhz * 1e6
    rate = pairs / (ms * 1e-3)
    return {"exp_per_s": float("%.4g" % rate), "mufu_peak_per_s": float("%.4g" % peak),
            "frac": round(rate / peak, 4), "sm_mhz": mhz}


def aggregate_tflops(flop_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: every rank does one replica's work per step."""
    return flop_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def bench_config(workload: str, det: bool, world: int) -> dict:
    """The `config` object of both arms' lines: the workload, its sizes and the step."""
    w = syn.WORKLOADS[workload]
    return {"workload": f"{workload}: {w.description}", "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "mask": w.mask, "step": "fa_fwd + " + ("fa_bwd_deterministic" if det else "fa_bwd"),
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: Q,K,V,dO are 4 x %.0f MiB per step"
                  % (w.B * w.H * w.N * w.d * 2 / 2**20)}


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank: int, world: int, dist):
    import exact_io_aware_98_b200 as fa
    fa.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    x = syn.workload_inputs(args.workload)
    H = x["q"].shape[1]
    B, N, d = x["B"], x["N"], x["d"]
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in x.items()}
    f_fwd, f_bwd = flops(x, H)
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(g["q"]) for _ in range(3))
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    kw = dict(scale=g["scale"], causal=g["causal"], block_mask=g["block_mask"],
              kv_len=g["kv_len"])

    det = bool(args.deterministic)

    def step():
        fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], workspace=ws, dq=dq, dk=dk, dv=dv,
               deterministic=det, **kw)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if fa.device_status() != 0:
        raise RuntimeError("a device-side wait gave up during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(dev.index)
    fa.kernel_timing_read("")  # forget anything recorded before the timed region
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = fa.launch_count()
    fa.kernel_timing(True)
    sampler.start()
    for s in range(K):
        ev[s][0].record()
        fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)
        ev[s][1].record()
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], workspace=ws, dq=dq, dk=dk, dv=dv,
               deterministic=det, **kw)
        ev[s][2].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    fa.kernel_timing(False)
    launches = fa.launch_count() - launches0
    bwd_kernels = (["fa_bwd_dkdv_sm100_kernel", "fa_bwd_dq_sm100_kernel"] if det
                   else ["fa_bwd_sm100_kernel"])
    kern = {name: fa.kernel_timing_read(name) for name in ["fa_fwd_sm100_kernel", *bwd_kernels]}
    if dist is not None:
        dist.barrier()
    total_ms = ev[0][0].elapsed_time(ev[K - 1][2])
    fwd_all = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_all = [e[1].elapsed_time(e[2]) for e in ev]
    fwd_ms, bwd_ms = statistics.mean(fwd_all), statistics.mean(bwd_all)
    total_ms, fwd_ms, bwd_ms = max_over_ranks([total_ms, fwd_ms, bwd_ms], dist, dev)
    status = fa.device_status()

    # ---- end to end through the public API: pinned host inputs in, results back to host
    e2e = None
    if not args.no_e2e:
        e2e = e2e_measurement(fa, x, g, kw, ws, det, B, H, N, f_fwd + f_bwd, K, world, dist, dev)

    ms_step = total_ms / K
    value = aggregate_tflops(f_fwd + f_bwd, world, ms_step)
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak, why = select_peak(peaks, clocks)
    fwd_tf = f_fwd / (fwd_ms * 1e-3) / 1e12
    bwd_tf = f_bwd / (bwd_ms * 1e-3) / 1e12
    # per-launch kernel durations, CUDA events on the launching stream inside the timed region
    names = list(kern)
    per = max_over_ranks([kern[n][1] / kern[n][0] if kern[n][0] else 0.0 for n in names],
                         dist, dev)
    k_ms = {n: (v if v > 0 else None) for n, v in zip(names, per)}
    fwd_k_ms = k_ms["fa_fwd_sm100_kernel"]
    bwd_k_ms = sum(k_ms[n] for n in bwd_kernels) if all(k_ms[n] for n in bwd_kernels) else None

    def fractions(tf):
        return {"frac_of_peak": round(tf / peak, 4), "frac_of_burst": round(tf / burst, 4),
                "frac_of_nominal_2250": round(tf / NOMINAL_BF16_TFLOPS, 4)}
    bwd_dom = bwd_ms >= fwd_ms
    dom_name = " + ".join(bwd_kernels) if bwd_dom else "fa_fwd_sm100_kernel"
    dom_flop = f_bwd if bwd_dom else f_fwd
    dom_kms = bwd_k_ms if bwd_dom else fwd_k_ms
    dom_call_tf = bwd_tf if bwd_dom else fwd_tf
    dom_tf = dom_flop / (dom_kms * 1e-3) / 1e12 if dom_kms else dom_call_tf
    if bwd_dom:
        parts = [traffic_for(k, args.workload) for k in bwd_kernels]
        traffic = None if any(t is None for t in parts) else sum(parts)
    else:
        traffic = traffic_for("fa_fwd_sm100_kernel", args.workload)
    roof = {"bound": "tensor", "kernel": dom_name, "achieved": round(dom_tf, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(dom_tf / peak, 4),
            "peak_source": f"{peak_src} {why}",
            "frac_of_burst": round(dom_tf / burst, 4),
            "frac_of_nominal_2250": round(dom_tf / NOMINAL_BF16_TFLOPS, 4),
            "kernel_ms": round(dom_kms, 4) if dom_kms else None,
            "call": {"ms": round(bwd_ms if bwd_dom else fwd_ms, 4),
                     "achieved": round(dom_call_tf, 2), **fractions(dom_call_tf)},
            "flop_per_launch": dom_flop, "traffic": traffic,
            "note": "achieved = algorithmic FLOP per launch (10 d per unmasked pair backward, 4 d "
                    "forward) / the kernel's mean launch duration, CUDA events recorded by the "
                    "library on the launching stream around each launch in the timed region; "
                    "`call` is the same over the whole entry-point call (the backward's "
                    "preprocess and dQ-convert launches included); traffic = ncu DRAM bytes of "
                    "the kernel launch(es) named in `kernel`"}
    target = {"fwd_frac_of_nominal": 0.60, "bwd_frac_of_nominal": 0.45,
              "fwd_frac_of_nominal_now": round((f_fwd / (fwd_k_ms * 1e-3) / 1e12 if fwd_k_ms
                                                else fwd_tf) / NOMINAL_BF16_TFLOPS, 4),
              "bwd_frac_of_nominal_now": round(bwd_tf / NOMINAL_BF16_TFLOPS, 4),
              "note": "targets at N >= 4096, d = 128 against the nominal 2.25 PFLOP/s dense "
                      "bf16; forward by its kernel, backward by its whole call"}
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1); Q,K x2), no dataset",
        "config": bench_config(args.workload, det, world),
        "fwd": {"ms": round(fwd_ms, 4), "tflops": round(fwd_tf, 2), **fractions(fwd_tf),
                "kernel_ms": round(fwd_k_ms, 4) if fwd_k_ms else None,
                "kernel_tflops": round(f_fwd / (fwd_k_ms * 1e-3) / 1e12, 2) if fwd_k_ms else None,
                **step_stats(fwd_all),
                "exp_roof": exp_roof(f_fwd / (4.0 * d), fwd_ms, clocks.get("sm_mhz"))},
        "bwd": {"ms": round(bwd_ms, 4), "tflops": round(bwd_tf, 2), **fractions(bwd_tf),
                "kernel_ms": round(bwd_k_ms, 4) if bwd_k_ms else None,
                "kernel_tflops": round(f_bwd / (bwd_k_ms * 1e-3) / 1e12, 2) if bwd_k_ms else None,
                **step_stats(bwd_all),
                "exp_roof": exp_roof(f_bwd / (10.0 * d), bwd_ms, clocks.get("sm_mhz"))},
        "roofline": roof,
        "target": target,
        "clocks": clocks,
        # counted by the library (fa_launch_count) over the timed region
        "gpu_launches": int(launches),
        "device_status": status,
        "e2e": e2e,
    }
    return line, (x, g, o, lse, dq)


def e2e_measurement(fa, x, g, kw, ws, det, B, H, N, flop, K, world, dist, dev):
    """The step through the public API with host buffers: every step copies its Q, K, V, dO
    from pinned host memory to the device and its O, lse, dQ, dK, dV back.

    Two schedules are timed.  Serial: copy in, fa_fwd + fa_bwd, copy out, all on one stream.
    Pipelined (the reported value): the copies run on their own streams with two device buffer
    sets, so step k+1's host-to-device copies and step k-1's device-to-host copies overlap step
    k's kernels; events order each buffer's reuse.  Both move the same bytes per step."""
    names_in = ("q", "k", "v", "do")
    hin = {k: x[k].pin_memory() for k in names_in}
    outs = (("o", g["q"].shape, g["q"].dtype), ("lse", (B, H, N), torch.float32),
            ("dq", g["q"].shape, g["q"].dtype), ("dk", g["k"].shape, g["k"].dtype),
            ("dv", g["v"].shape, g["v"].dtype))
    nb = 2
    din = [{k: torch.empty_like(g[k]) for k in names_in} for _ in range(nb)]
    dout = [{n: torch.empty(shp, dtype=dt, device=dev) for n, shp, dt in outs} for _ in range(nb)]
    hout = [{n: torch.empty(shp, dtype=dt).pin_memory() for n, shp, dt in outs} for _ in range(nb)]
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = sum(t.numel() * t.element_size() for t in hout[0].values())

    def compute(di, do_):
        fa.fwd(di["q"], di["k"], di["v"], out=do_["o"], lse=do_["lse"], **kw)
        fa.bwd(di["q"], di["k"], di["v"], do_["o"], do_["lse"], di["do"], workspace=ws,
               dq=do_["dq"], dk=do_["dk"], dv=do_["dv"], deterministic=det, **kw)

    def serial_step():
        for k in names_in:
            din[0][k].copy_(hin[k], non_blocking=True)
        compute(din[0], dout[0])
        for n, _, _ in outs:
            hout[0][n].copy_(dout[0][n], non_blocking=True)

    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def pipelined(steps, e0, e1):
        ev_in = [torch.cuda.Event() for _ in range(steps)]
        ev_cmp = [torch.cuda.Event() for _ in range(steps)]
        ev_out = [torch.cuda.Event() for _ in range(steps)]
        e0.record(s_in)
        s_cmp.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(steps):
            b = i % nb
            with torch.cuda.stream(s_in):
                if i >= nb:
                    s_in.wait_event(ev_cmp[i - nb])   # step i-2's kernels are done with din[b]
                for k in names_in:
                    din[b][k].copy_(hin[k], non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if i >= nb:
                    s_cmp.wait_event(ev_out[i - nb])  # step i-2's results have left dout[b]
                compute(din[b], dout[b])
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                for n, _, _ in outs:
                    hout[b][n].copy_(dout[b][n], non_blocking=True)
                ev_out[i].record(s_out)
        e1.record(s_out)

    Ke = max(3, min(K, 10))
    res = {}
    for mode in ("serial", "pipelined"):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if mode == "serial":
            serial_step()
        else:
            pipelined(2, torch.cuda.Event(), torch.cuda.Event())
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        if mode == "serial":
            e0.record()
            for _ in range(Ke):
                serial_step()
            e1.record()
        else:
            pipelined(Ke, e0, e1)
        torch.cuda.synchronize()
        res[mode] = max_over_ranks([e0.elapsed_time(e1)], dist, dev)[0] / Ke
    if fa.device_status() != 0:
        raise RuntimeError("a device-side wait gave up in the end-to-end runs")
    ms_e = res["pipelined"]
    return {"value": round(aggregate_tflops(flop, world, ms_e), 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms_e, 4), "steps": Ke,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "mode": "pipelined: step k+1's H2D copies and step k-1's D2H copies overlap step "
                    "k's kernels on separate streams (two device buffer sets)",
            "serial": {"value": round(aggregate_tflops(flop, world, res["serial"]), 3),
                       "ms_per_step": round(res["serial"], 4)}}


# ----------------------------------------------------------------------------- CPU baseline leg
def cpu_baseline_leg(args, x, o, lse, dq):
    """Times the FP64 oracle on a bounded row sample of the same workload on this host's cores
    and, from the same oracle results, reports the GPU outputs' error on those rows."""
    import oracle
    N, H, d = x["N"], x["q"].shape[1], x["d"]
    xd = {k: x[k].double().numpy() for k in ("q", "k", "v", "do")}  # widened once, untimed
    rng = np.random.default_rng(1234)
    rows = np.sort(rng.choice(x["B"] * H * N, size=min(args.cpu_rows, x["B"] * H * N),
                              replace=False))
    t0 = time.perf_counter()
    o_ref, l_ref = oracle.attn_fwd_rows(xd["q"], xd["k"], xd["v"], x["scale"], rows,
                                        x["causal"], x["block_mask"], x["kv_len"])
    dq_ref = oracle.attn_bwd_dq_rows(xd["q"], xd["k"], xd["v"], xd["do"], x["scale"], rows,
                                     x["causal"], x["block_mask"], x["kv_len"])
    dt = time.perf_counter() - t0
    n = row_pairs(x, rows)
    fl = 10.0 * d * n.sum()   # forward 4 d n_i + recompute S, dP and dQ 6 d n_i
    o_g = o.float().cpu().double().numpy().reshape(-1, d)[rows]
    l_g = lse.float().cpu().double().numpy().reshape(-1)[rows]
    dq_g = dq.float().cpu().double().numpy().reshape(-1, d)[rows]
    eo = np.abs(o_g - o_ref)
    fin = np.isfinite(l_ref)
    el = np.abs(l_g[fin] - l_ref[fin]) if fin.any() else np.zeros(1)
    edq = np.abs(dq_g - dq_ref) / max(np.abs(dq_ref).max(), 1e-30)
    cpu = {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
           "kind": "oracle",
           "sample": f"O, lse and dQ of {len(rows)} random query rows of {args.workload} "
                     f"(FP64, S and A rows materialised); {dt:.1f} s wall",
           "seconds": round(dt, 2)}
    err = {"rows": len(rows), "o_max": float(eo.max()), "o_mean": float(eo.mean()),
           "lse_max": float(el.max()), "dq_max_rel": float(edq.max()),
           "dq_mean_rel": float(edq.mean()),
           "tolerance": "O: max 2e-2, mean 2e-3; dQ: same relative to max|ref|"}
    return cpu, err


def deviation_sweep():
    """Numeric deviation vs the FP64 golden across key-tile widths, next to the naive kernel
    (the microbenchmark of "Is Flash Attention Stable?"), on 32 heads of the padding workload.
    Each variant is measured on its bf16 output and, beside it, on the fp32 O/l before that
    rounding: the bf16 cast alone contributes up to half an ulp of O, which would otherwise hide
    the effect of the tile width."""
    import oracle
    import exact_io_aware_98_b200 as fa
    x = syn.workload_inputs("bert_padding", with_grad=False, H=2)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    gold, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], x["scale"], False, None, x["kv_len"])
    out = {}

    def stat(t):
        e = np.abs(t.float().cpu().double().numpy() - gold)
        return {"max": float(e.max()), "mean": float(e.mean())}

    def both(**kw_tile):
        o, _ = fa.fwd_tile_reference(g["q"], g["k"], g["v"], scale=g["scale"], kv_len=g["kv_len"],
                                     **kw_tile)
        o32, _ = fa.fwd_tile_reference(g["q"], g["k"], g["v"], scale=g["scale"],
                                       kv_len=g["kv_len"], o_f32=True, **kw_tile)
        return {"bf16": stat(o), "fp32_before_cast": stat(o32)}
    # the tensor-core forward itself at two key-tile widths (64 is the library's d = 64 kernel)
    for bc in (64, 128):
        out[f"tcgen05_Br128_Bc{bc}_lazy"] = both(bc=bc, tensor_core=True)
    # the study's axes on the CUDA-core reference: key-tile width Bc, the order the key tiles are
    # visited in, and whether the normaliser l sums the fp32 P or the bf16-rounded P
    for bc in (64, 128, 256):
        for reverse in (False, True):
            for l_rounded in (False, True):
                key = f"tile_Bc{bc}_{'reverse' if reverse else 'forward'}_l{'bf16' if l_rounded else 'fp32'}"
                out[key] = both(bc=bc, reverse=reverse, l_rounded=l_rounded)
    kw = dict(scale=g["scale"], kv_len=g["kv_len"])
    o_n, _ = fa.naive_fwd(g["q"], g["k"], g["v"], **kw)
    out["naive_materialised"] = {"bf16": stat(o_n)}
    o_tc, _ = fa.fwd(g["q"], g["k"], g["v"], **kw)
    diff = (o_tc.float() - o_n.float()).abs()
    out["tcgen05_vs_naive"] = {"max": float(diff.max()), "mean": float(diff.mean())}
    out["note"] = ("row-wise arithmetic does not depend on Br (query-tile height), so the sweep "
                   "varies Bc; the tcgen05 kernel is Br=128 with a lazy (2^8) rescale")
    return out


def workload_measurement(name: str, iters: int = 20, flush_bytes: int = 256 << 20) -> dict:
    """fa_fwd and fa_bwd on one of the other workloads: CUDA events per call, then, in a second
    pass, each tensor-core kernel's own launches (events the library records around them; those
    events are recorded between the backward's launches and can stop them overlapping, so the
    calls are timed without them).  These inputs fit in L2, so a buffer larger than L2 is overwritten before
    every step."""
    import exact_io_aware_98_b200 as fa
    w = syn.WORKLOADS[name]
    x = syn.workload_inputs(name)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    H = x["q"].shape[1]
    B, N, d = x["B"], x["N"], x["d"]
    f_fwd, f_bwd = flops(x, H)
    kw = dict(scale=g["scale"], causal=g["causal"], block_mask=g["block_mask"],
              kv_len=g["kv_len"])
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device="cuda")
    res = {"config": w.description, "dtype": w.dtype,
           "l2": f"{flush_bytes >> 20} MiB overwritten before every step (inputs fit in L2)"}
    if not w.backward:
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
        for _ in range(3):
            fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)
        for e in ev:
            flush.zero_()
            e[0].record()
            fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)
            e[1].record()
        torch.cuda.synchronize()
        ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
        res["fwd"] = {"median_ms": round(ms, 5), "gflops": round(f_fwd / ms / 1e6, 3),
                      "note": "CUDA-core fp32 kernel; latency-bound at this size, no roofline"}
        res["device_status"] = fa.device_status()
        return res
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    dq, dk, dv = (torch.empty_like(g["q"]) for _ in range(3))

    def fwd():
        fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)

    def bwd():
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], workspace=ws, dq=dq, dk=dk, dv=dv, **kw)
    for _ in range(3):
        fwd()
        bwd()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(iters)]
    for e in ev:
        flush.zero_()
        e[0].record()
        fwd()
        e[1].record()
        bwd()
        e[2].record()
    torch.cuda.synchronize()
    fa.kernel_timing_read("")
    fa.kernel_timing(True)
    for _ in range(iters):
        flush.zero_()
        fwd()
        bwd()
    torch.cuda.synchronize()
    fa.kernel_timing(False)
    peaks, _ = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    for key, flop, i0, i1, kname in (("fwd", f_fwd, 0, 1, "fa_fwd_sm100_kernel"),
                                     ("bwd", f_bwd, 1, 2, "fa_bwd_sm100_kernel")):
        ms = statistics.median(e[i0].elapsed_time(e[i1]) for e in ev)
        n, kms = fa.kernel_timing_read(kname)
        kms = kms / n if n else None
        tf = flop / ms / 1e9
        res[key] = {"median_ms": round(ms, 5), "tflops": round(tf, 2),
                    "frac_of_burst": round(tf / burst, 4),
                    "kernel_ms": round(kms, 5) if kms else None,
                    "kernel_tflops": round(flop / kms / 1e9, 2) if kms else None,
                    "kernel_frac_of_burst": round(flop / kms / 1e9 / burst, 4) if kms else None,
                    "flop": flop}
    res["device_status"] = fa.device_status()
    return res


def deterministic_measurement(x, g, o, lse, iters: int = 10):
    """fa_bwd_deterministic on the bench workload: dQ from the query-stationary kernel, no
    atomics.  Reported against the same algorithmic backward FLOPs (10 d per pair) as fa_bwd,
    and against the FLOPs it executes (14 d per pair: S and dP are computed twice)."""
    import exact_io_aware_98_b200 as fa
    H = x["q"].shape[1]
    B, N, d = x["B"], x["N"], x["d"]
    _, f_bwd = flops(x, H)
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=g["q"].device)
    dq, dk, dv = (torch.empty_like(g["q"]) for _ in range(3))
    kw = dict(scale=g["scale"], causal=g["causal"], block_mask=g["block_mask"],
              kv_len=g["kv_len"], workspace=ws, dq=dq, dk=dk, dv=dv, deterministic=True)
    for _ in range(3):
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], **kw)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], **kw)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    return {"ms": round(ms, 4), "tflops_algorithmic": round(f_bwd / ms / 1e9, 2),
            "tflops_executed": round(1.4 * f_bwd / ms / 1e9, 2),
            "device_status": fa.device_status(),
            "note": "dK/dV by fa_bwd_dkdv_sm100_kernel, dQ by fa_bwd_dq_sm100_kernel"}


def gqa_measurement(iters: int = 10):
    """Grouped-query attention (the MQA/GQA of the tcdigital FA-2 ROI article) on a Llama-class
    grouping: B1 H32 H_kv8 N8192 d128 causal.  FLOPs count per query head, as for attention with
    H heads; the K/V reads shrink by H/H_kv."""
    import exact_io_aware_98_b200 as fa
    B, H, H_kv, N, d = 1, 32, 8, 8192, 128
    x = syn.make_inputs(B, H, N, d, "bf16", seed=1400, qk_amp=2.0, causal=True, H_kv=H_kv)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    f_fwd, f_bwd = flops(x, H)
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    kw = dict(scale=g["scale"], causal=True)
    for _ in range(3):
        fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], workspace=ws, dq=dq, dk=dk, dv=dv, **kw)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    for _ in range(iters):
        fa.fwd(g["q"], g["k"], g["v"], out=o, lse=lse, **kw)
    ev[1].record()
    for _ in range(iters):
        fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], workspace=ws, dq=dq, dk=dk, dv=dv, **kw)
    ev[2].record()
    torch.cuda.synchronize()
    fwd_ms, bwd_ms = ev[0].elapsed_time(ev[1]) / iters, ev[1].elapsed_time(ev[2]) / iters
    return {"config": f"B{B} H{H} H_kv{H_kv} N{N} d{d} causal, bf16 (Q,K x2)",
            "fwd": {"ms": round(fwd_ms, 4), "tflops": round(f_fwd / fwd_ms / 1e9, 2)},
            "bwd": {"ms": round(bwd_ms, 4), "tflops": round(f_bwd / bwd_ms / 1e9, 2)},
            "device_status": fa.device_status()}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, world: int):
    import oracle
    x = syn.workload_inputs(args.workload)
    N, H, d = x["N"], x["q"].shape[1], x["d"]
    xd = {k: x[k].double().numpy() for k in ("q", "k", "v", "do")}  # widened once, untimed
    rng = np.random.default_rng(99)
    R = min(args.ref_rows, x["B"] * H * N)

    def one(seed):
        rows = np.sort(np.random.default_rng(seed).choice(x["B"] * H * N, size=R, replace=False))
        t0 = time.perf_counter()
        oracle.attn_fwd_rows(xd["q"], xd["k"], xd["v"], x["scale"], rows, x["causal"],
                             x["block_mask"], x["kv_len"])
        oracle.attn_bwd_dq_rows(xd["q"], xd["k"], xd["v"], xd["do"], x["scale"], rows,
                                x["causal"], x["block_mask"], x["kv_len"])
        return time.perf_counter() - t0, 10.0 * d * row_pairs(x, rows).sum()

    for w in range(args.warmup):
        one(int(rng.integers(1 << 30)))
    tt, ff = 0.0, 0.0
    for s in range(args.steps):
        dt, fl = one(int(rng.integers(1 << 30)))
        tt += dt
        ff += fl
    value = ff / tt / 1e12
    sample = f"O, lse and dQ of {R} random query rows of {args.workload} per step (FP64)"
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(args.workload, False, world),
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                             "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    dist = init_distributed("nccl")
    try:
        line, (x, g, o, lse, dq) = run_ours(args, rank, world, dist)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cpu, err = cpu_baseline_leg(args, x, o, lse, dq)
            line["cpu_baseline"] = cpu
            line["max_err_vs_fp64"] = err
            line["deviation_sweep"] = deviation_sweep()
            line["bwd_deterministic"] = deterministic_measurement(x, g, o, lse)
            line["gqa"] = gqa_measurement()
            line["workloads"] = {n: workload_measurement(n) for n in
                                 ("gpt2_causal", "bert_padding", "block_sparse",
                                  "fp32_single_head")}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
