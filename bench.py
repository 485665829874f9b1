#!/usr/bin/env python
"""Throughput of the causal FFT long convolution on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one forward pass of the whole hot path (load, FFT, product with the
cached kernel spectrum, inverse FFT, truncation, skip term / gate, store) over
one batch of the named synthetic workload.  The kernel spectrum is computed
once per plan, before timing.  Default workload: B=8, H=768, N=4096, bf16
(the Hyena-style layer convolution).

Timing: W untimed warm-up steps; then a barrier and a device synchronise; then
exactly K steps, each bracketed by CUDA events on the launching stream with an
L2 flush (a 256 MiB write, more than the 126 MB L2) between steps outside the
events; a synchronise and a barrier; the max over ranks.  value = outputs of
all ranks / that time (weak scaling: every rank runs the full workload; the
rows are independent so no collective is on the data path).

e2e: the same step through the public API from pinned host buffers, with the
host->device copy of the inputs and the device->host copy of y inside the
timed region; steps of 1 MiB of input or more alternate between two streams
with their own buffers, so one step's input copy overlaps the previous step's
output copy.

cpu_baseline (rank 0, N=1): the CPU fp64 oracle, as it stands, on a bounded
uniform sample of the same workload's outputs.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FFT-conv output elems/s and % of HBM roofline (1 B200), N=1K–1M and 2-D"
DEFAULT_CONFIG = "hyena_b8_h768_n4096_bf16"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
KERNEL_SOURCES = ["fft_simt.cuh", "conv1d_simt.cu", "conv2d_simt.cu", "tc_common.cuh", "conv1d_mma.cu", "umma.cuh",
                  "conv1d_umma.cu", "conv2d_tc.cu"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--channels", type=int, default=0,
                    help="override H (1-D) or C (2-D) for a smaller case, e.g. an ncu capture; 0 = as named")
    return ap.parse_args()


def dist_env():
    from fft_long_convolution_causal_b200.dist import rank_env
    return rank_env()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            d = json.load(open(path))
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "fft_long_convolution_causal_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(config, kernel):
    """DRAM bytes per launch from a committed ncu summary, if it still matches the sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        d = json.load(open(path))
        e = d.get(config, {})
        if e.get("kernel") == kernel and e.get("source_hash") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fftconv_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        load = [r for r in rows if r["power"] > 300.0] or rows
        return {"sm_mhz": float(np.median([r["sm"] for r in load])), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# --------------------------------------------------------------- workload
def build_workload(name, channels=0):
    from fft_long_convolution_causal_b200 import workloads
    if not channels:
        return workloads.make_config(name)
    c = dict(workloads.CONFIGS[name])
    kind = c.pop("kind")
    if kind == "1d":
        c["H"] = channels
        return workloads.make_1d(name=f"{name}_h{channels}", **c)
    c["C"] = channels
    return workloads.make_2d(name=f"{name}_c{channels}", **c)


class Runner:
    """Device-resident workload + plan; step() enqueues one forward."""

    def __init__(self, wl, torch):
        from fft_long_convolution_causal_b200 import binding
        self.torch = torch
        self.wl = wl
        dev = torch.device("cuda")
        tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.tdt = tdt

        def up(a):
            return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev, tdt)

        self.is2d = hasattr(wl, "C")
        if self.is2d:
            self.plan = binding.Plan2D(wl.B, wl.C, wl.Hs, wl.Ws, wl.dtype)
            self.khat = self.plan.kernel_spectrum(torch.from_numpy(wl.k).to(dev))
            self.u = up(wl.u)
            self.v = self.w = self.D = None
            self.y = torch.empty_like(self.u)
            self.outputs = wl.B * wl.C * wl.Hs * wl.Ws
        else:
            self.plan = binding.Plan(wl.B, wl.H, wl.N, wl.dtype, gated=wl.gated)
            self.khat = self.plan.kernel_spectrum(torch.from_numpy(wl.k).to(dev))
            self.u, self.v, self.w = up(wl.u), up(wl.v), up(wl.w)
            self.D = None if wl.D is None else torch.from_numpy(wl.D).to(dev)
            self.y = torch.empty_like(self.u)
            self.outputs = wl.B * wl.H * wl.N
        self.ws = self.plan.new_workspace()
        torch.cuda.synchronize()

    def step(self, y=None, u=None, v=None, w=None, ws=None):
        y = self.y if y is None else y
        u = self.u if u is None else u
        ws = self.ws if ws is None else ws
        if self.is2d:
            self.plan.fwd(u, self.khat, y=y, workspace=ws)
        else:
            self.plan.fwd(u, self.khat, D=self.D, v=self.v if v is None else v, w=self.w if w is None else w,
                          y=y, workspace=ws)

    def launches_per_step(self):
        if self.plan.path in ("fused", "fused_tc", "fused_umma"):
            return 1
        pairs = ((self.wl.B + 1) // 2) * (self.wl.C if self.is2d else self.wl.H)
        group = max(1, self.plan.workspace_bytes // self._pair_bytes())
        return 3 * int(np.ceil(pairs / group))

    def _pair_bytes(self):
        if self.is2d:
            return self.wl.Hs * 2 * self.wl.Ws * 8
        return 2 * self.wl.N * 8

    def compute_dtype(self):
        return {"fused": "f32", "multipass": "f32", "2d": "f32", "fused_tc": "bf16",
                "fused_umma": "bf16", "2d_tc": "f32+bf16"}.get(self.plan.path, "f32")

    def dominant_kernel(self):
        return {"fused": "fused_fwd_simt", "multipass": "mp_pass2", "2d": "c2_pass2",
                "fused_tc": "fused_fwd_tc", "fused_umma": "fused_fwd_umma", "2d_tc": "c2tc_cols"}.get(self.plan.path)


def time_steps(r, steps, torch, flush):
    """Per-step device time (ms) with an L2 flush between steps outside the events."""
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush.fill_(1)
        a.record(stream)
        r.step()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_e2e(r, steps, torch):
    """Host buffers in, host buffer out, copies inside the timed region.

    Steps of at least 1 MiB of input alternate between two CUDA streams,
    each with its own device buffers, workspace and pinned output buffer
    (double buffering, as a streaming caller would run it): step i+1's
    host-to-device copy overlaps step i's device-to-host copy on the
    full-duplex link.  Smaller steps, bound by per-call latency, run on the
    current stream alone.  Every step copies all of its inputs in and its
    whole result out."""
    pin = lambda t: None if t is None else t.cpu().pin_memory()  # noqa: E731
    hu, hv, hw = pin(r.u), pin(r.v), pin(r.w)
    h2d = sum(t.numel() * t.element_size() for t in (hu, hv, hw) if t is not None)
    main = torch.cuda.current_stream()
    nsets = 2 if h2d >= (1 << 20) else 1
    sets = []
    for _ in range(nsets):
        sets.append(dict(
            du=torch.empty_like(r.u), dy=torch.empty_like(r.y),
            dv=None if r.v is None else torch.empty_like(r.v), dw=None if r.w is None else torch.empty_like(r.w),
            ws=r.plan.new_workspace(), hy=torch.empty(r.y.shape, dtype=r.y.dtype).pin_memory(),
            stream=torch.cuda.Stream() if nsets > 1 else main))
    d2h = sets[0]["hy"].numel() * sets[0]["hy"].element_size()

    def one(i):
        b = sets[i % nsets]
        with torch.cuda.stream(b["stream"]):
            b["du"].copy_(hu, non_blocking=True)
            if b["dv"] is not None:
                b["dv"].copy_(hv, non_blocking=True)
                b["dw"].copy_(hw, non_blocking=True)
            r.step(y=b["dy"], u=b["du"], v=b["dv"], w=b["dw"], ws=b["ws"])
            b["hy"].copy_(b["dy"], non_blocking=True)

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for b in sets:
        if b["stream"] is not main:
            b["stream"].wait_event(a)
    for i in range(steps):
        one(i)
    for b in sets:
        if b["stream"] is not main:
            main.wait_stream(b["stream"])
    e.record(main)
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / steps
    return ms, h2d, d2h


# ------------------------------------------------------------ CPU oracle
class OracleSampler:
    """Times the fp64 oracle on uniform samples of the workload's outputs."""

    def __init__(self, wl, seed=0):
        import oracle
        self.oracle = oracle
        self.wl = wl
        self.rng = np.random.default_rng(seed)
        self.is2d = hasattr(wl, "C")
        self.total = (wl.B * wl.C * wl.Hs * wl.Ws) if self.is2d else (wl.B * wl.H * wl.N)
        oracle.num_threads()  # builds and loads the oracle outside any timing

    def run(self, n):
        wl, rng, o = self.wl, self.rng, self.oracle
        if self.is2d:
            idx = (rng.integers(0, wl.B, n), rng.integers(0, wl.C, n), rng.integers(0, wl.Hs, n),
                   rng.integers(0, wl.Ws, n))
            t0 = time.perf_counter()
            o.causal_conv2d_points(wl.u, wl.k, *idx)
        else:
            b, h, t = rng.integers(0, wl.B, n), rng.integers(0, wl.H, n), rng.integers(0, wl.N, n)
            t0 = time.perf_counter()
            o.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D, w=wl.w, v=wl.v)
        return time.perf_counter() - t0

    def calibrate(self, target_s):
        """Sample size whose oracle run takes about target_s seconds."""
        n = 256
        dt = self.run(n)
        while dt < 0.25 and n < 1 << 26:
            n *= 4
            dt = self.run(n)
        return int(min(max(n * target_s / max(dt, 1e-6), 64), self.total))

    def describe(self, n, dt):
        return (f"{n} uniformly drawn outputs of {self.total} (direct fp64 sum per output), "
                f"{dt:.1f} s")


def cpu_oracle_rate(wl, target_s, seed=0):
    """Outputs/s of the fp64 oracle on a uniform sample of the workload's outputs."""
    s = OracleSampler(wl, seed)
    n = s.calibrate(target_s)
    dt = s.run(n)
    return {"value": n / dt, "unit": "elems/s", "cores": s.oracle.num_threads(), "kind": "oracle",
            "sample": s.describe(n, dt)}


# ------------------------------------------------------------------ main
def main():
    args = parse()
    rank, world, local = dist_env()
    import torch
    if args.impl == "reference":
        return main_reference(args, rank, world)
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        pg = dist
    wl = build_workload(args.config, args.channels)
    r = Runner(wl, torch)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    for _ in range(max(args.warmup, 3)):
        r.step()
    torch.cuda.synchronize()
    sampler = None if (args.no_clocks or rank != 0) else ClockSampler(local)
    if sampler:
        sampler.start()
        # keep the GPU busy for a moment so the clock samples see it under load
        t_end = time.time() + 0.6
        while time.time() < t_end:
            for _ in range(20):
                flush.fill_(1)
                r.step()
            torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    per_step = time_steps(r, args.steps, torch, flush)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clocks = sampler.stop() if sampler else None
    from fft_long_convolution_causal_b200.dist import job_throughput, max_over_ranks
    total_ms = max_over_ranks(float(np.sum(per_step)), pg, device="cuda")
    ms_per_step = total_ms / args.steps
    value = job_throughput(r.outputs, world, ms_per_step * 1e-3)

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = time_e2e(r, max(3, min(args.steps, 20)), torch)
        e2e_ms = max_over_ranks(e2e_ms, pg, device="cuda")
        e2e = {"value": job_throughput(r.outputs, world, e2e_ms * 1e-3), "unit": "elems/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    peak, peak_kind = measured_peaks()
    alg_bytes = wl.io_bytes()
    launches = r.launches_per_step()
    # The fused path is one launch per step, so the step's event time is that
    # kernel's time; for multi-launch paths the whole step is charged to the
    # dominant kernel (a lower bound on its achieved rate).
    achieved = alg_bytes / (ms_per_step * 1e-3) / 1e9
    kname = r.dominant_kernel()
    traffic = recorded_traffic(args.config, kname)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kname,
                "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": alg_bytes}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_rate(wl, args.cpu_seconds)

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg = {"workload": wl.name, "dtype_io": wl.dtype, "path": r.plan.path,
           "l2": "flushed between timed steps (256 MiB write outside the events)",
           "parallelism": f"replicas x{world} (independent rows, no collective)"}
    if r.is2d:
        cfg.update(B=wl.B, C=wl.C, Hs=wl.Hs, Ws=wl.Ws)
    else:
        cfg.update(B=wl.B, H=wl.H, N=wl.N, gated=wl.gated, skip_term=wl.D is not None)
    line = {"metric": METRIC, "value": value, "unit": "elems/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": r.compute_dtype(), "data": "synthetic", "config": cfg,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches * args.steps, "clocks": clocks,
            "ms_per_step_min": float(np.min(per_step)), "ms_per_step_median": float(np.median(per_step))}
    print(json.dumps(line))
    return 0


def main_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 times it on the host cores."""
    if rank != 0:
        return 0
    wl = build_workload(args.config, args.channels)
    s = OracleSampler(wl, seed=0)
    per_step = max(args.cpu_seconds / max(args.steps, 1), 0.25)
    n = s.calibrate(per_step)
    for _ in range(args.warmup):
        s.run(max(n // 8, 64))
    times = [s.run(n) for _ in range(args.steps)]
    value = n * len(times) / float(np.sum(times))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "elems/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s.total / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.config, "dtype_io": wl.dtype},
            "cpu_baseline": {"value": value, "unit": "elems/s", "cores": s.oracle.num_threads(), "kind": "oracle",
                             "sample": "each step: " + s.describe(n, float(np.mean(times)))},
            "e2e": {"value": value, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
