#!/usr/bin/env python
"""Throughput of the causal FFT long convolution on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one forward pass of the whole hot path (load, FFT, product with the
cached kernel spectrum, inverse FFT, truncation, skip term / gate, store) over
one batch of the named synthetic workload.  The kernel spectrum is computed
once per plan, before timing.  Default workload: B=8, H=768, N=4096, bf16
(the Hyena-style layer convolution); at one GPU the line also carries
`per_config`, the same measurement for each of the other named workloads
(N = 1K, 16K gated, 1M, and 2-D 256 x 256), fewer steps each.

Timing: W untimed warm-up steps; then a barrier and a device synchronise; then
exactly K steps, each bracketed by CUDA events on the launching stream with an
L2 flush (a 256 MiB write, more than the 126 MB L2) between steps outside the
events; a synchronise and a barrier; the max over ranks.  value = outputs of
all ranks / that time.

Several GPUs (torchrun, one rank per GPU): the channels are sharded, one
contiguous block per rank, with no collective on the data path (rows are
independent and every channel's spectrum is read-only).  --shard weak
(default): the job at N ranks is the named workload with N times its channels,
rank r holding block r (the named shape per GPU; each rank draws its block
with its own seed).  --shard strong: the named workload's channels are split
over the ranks (total work fixed).

e2e: the same step through the public API from pinned host buffers, with the
host->device copy of the inputs and the device->host copy of y inside the
timed region; steps of 1 MiB of input or more alternate between two streams
with their own buffers, so one step's input copy overlaps the previous step's
output copy.

cpu_baseline (rank 0, N=1): the CPU fp64 oracle, as it stands, on a bounded
uniform sample of the same workload's outputs.

variants (N=1): the skipped-work forms on the long workload's shape, each
timed against the dense multi-pass plan on the same inputs (partial
convolution, frequency-sparse filter, state-space filters with chunked state
passing), the backward pass of the Hyena-style layer against its forward,
and the 3-D causal convolution on 64^3 fp32 volumes.
"""
import argparse
import hashlib
import json
import os
import re
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
# Source files each dominant kernel is built from: a recorded DRAM-traffic
# figure is valid only while the hash of these files matches.
# The translation unit of each dominant kernel; its sources are that file and
# every header under csrc/ it includes, directly or through other headers.
KERNEL_UNITS = {
    "fused_fwd_simt": "conv1d_simt.cu",
    "mp_pass2": "conv1d_simt.cu",
    "c2_pass2": "conv2d_simt.cu",
    "fused_fwd_tc": "conv1d_mma.cu",
    "fused_fwd_umma": "conv1d_umma.cu",
    "fused_fwd_t2": "conv1d_t2.cu",
    "c2tc_cols": "conv2d_tc.cu",
}
KERNEL_SOURCES = KERNEL_UNITS  # kernel names recognised in an ncu capture
CSRC = os.path.join(ROOT, "fft_long_convolution_causal_b200", "csrc")


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
    ap.add_argument("--shard", default="weak", choices=["weak", "strong"],
                    help="several GPUs: N x the channels (weak) or the named channels split (strong)")
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "mma_sync", "tcgen05"],
                    help="kernel family the plans may use (the library's choice by default)")
    ap.add_argument("--no-per-config", action="store_true", help="headline workload only")
    ap.add_argument("--per-config-steps", type=int, default=10)
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the partial / frequency-sparse / state-passing comparisons")
    ap.add_argument("--record-traffic", metavar="NCU_RAW_CSV",
                    help="write profiles/traffic.json's entry for --config from an ncu raw CSV and exit")
    ap.add_argument("--traffic-command", default="", help="the capture command, stored with the record")
    return ap.parse_args()


def dist_env():
    from fft_long_convolution_causal_b200.dist import rank_env
    return rank_env()


FALLBACK_BF16_TFLOPS = 1590.0


def measured_peaks():
    """(HBM GB/s, bf16 dense TFLOP/s burst, source) from MEASURED_PEAKS.json, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            d = json.load(open(path))
            return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def kernel_sources(kernel):
    """The kernel's translation unit and the csrc/ headers it includes,
    transitively, sorted.  The public API header (include/) declares entry
    points and status codes only and is not followed."""
    unit = KERNEL_UNITS.get(kernel)
    if unit is None:
        return []
    seen, todo = set(), [unit]
    while todo:
        f = todo.pop()
        path = os.path.join(CSRC, f)
        if f in seen or not os.path.exists(path):
            continue
        seen.add(f)
        todo += re.findall(r'#include "([^"]+)"', open(path, encoding="utf-8").read())
    return sorted(seen)


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    for f in kernel_sources(kernel):
        h.update(f.encode() + b"\0" + open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()[:16]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def recorded_traffic(config, kernel):
    """DRAM bytes per launch of `kernel` on `config` from the committed record,
    if the kernel's sources still hash to what they were when it was taken."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    try:
        e = json.load(open(TRAFFIC_JSON)).get(config, {})
        if e.get("kernel") == kernel and e.get("source_hash") == kernel_source_hash(kernel):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


def record_traffic(csv_path, config, channels, command):
    """Write profiles/traffic.json's entry for `config` from an ncu raw CSV
    (`ncu -i X.ncu-rep --page raw --csv`) of the config's dominant kernel.
    A capture on fewer channels (--channels) is scaled to the full workload by
    the channel ratio (each launch processes every channel once)."""
    import csv
    from fft_long_convolution_causal_b200 import workloads
    rows = list(csv.reader(open(csv_path)))
    head = rows[0]
    data = [r for r in rows[1:] if len(r) == len(head) and r[head.index("ID")].strip().isdigit()]
    kcol, rcol, wcol = head.index("Kernel Name"), head.index("dram__bytes_read.sum"), head.index("dram__bytes_write.sum")
    units = {rows[1][i] for i in (rcol, wcol)}

    def to_bytes(v, unit):
        f = float(v.replace(",", ""))
        return f * {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}.get(unit, 1)

    kname = data[0][kcol]
    short = next((k for k in KERNEL_SOURCES if k in kname), None)
    per = [to_bytes(r[rcol], rows[1][rcol]) + to_bytes(r[wcol], rows[1][wcol]) for r in data]
    c = workloads.CONFIGS[config]
    full = c["H"] if c["kind"] == "1d" else c["C"]
    scale = full / channels if channels else 1.0
    d = json.load(open(TRAFFIC_JSON)) if os.path.exists(TRAFFIC_JSON) else {}
    d[config] = {"kernel": short, "dram_bytes_per_launch": float(np.mean(per)) * scale,
                 "source_hash": kernel_source_hash(short), "launches_captured": len(per),
                 "captured_channels": channels or full, "scaled_by": scale, "units_seen": sorted(units),
                 "command": command}
    json.dump(d, open(TRAFFIC_JSON, "w"), indent=1, sort_keys=True)
    print(json.dumps(d[config]))


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
def build_workload(name, channels=0, rank=0, world=1, shard="weak"):
    """The named workload (or a smaller one with `channels`), as this rank's shard.

    weak: the rank's block of a job with world x the channels, drawn with the
    named seed + 1000 * rank (rank 0 draws exactly the named workload).
    strong: the named workload's channel block shard_channels(H, world, rank)."""
    from fft_long_convolution_causal_b200 import dist as fdist
    from fft_long_convolution_causal_b200 import workloads
    c = dict(workloads.CONFIGS[name])
    kind = c.pop("kind")
    label = name
    if channels:
        c["H" if kind == "1d" else "C"] = channels
        label = f"{name}_{'h' if kind == '1d' else 'c'}{channels}"
    if world > 1 and shard == "weak":
        c["seed"] = c["seed"] + 1000 * rank
    wl = workloads.make_1d(name=label, **c) if kind == "1d" else workloads.make_2d(name=label, **c)
    if world > 1 and shard == "strong":
        nch = wl.H if kind == "1d" else wl.C
        if nch < world:  # every rank reaches this, so all of them stop together
            raise SystemExit(f"--shard strong: {world} ranks for {nch} channels leaves ranks without work")
        a, b = fdist.shard_channels(nch, world, rank)
        wl = fdist.slice_channels_1d(wl, a, b) if kind == "1d" else fdist.slice_channels_2d(wl, a, b)
    return wl


class Runner:
    """Device-resident workload + plan; step() enqueues one forward."""

    def __init__(self, wl, torch, kernel="auto"):
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
            self.plan = binding.Plan2D(wl.B, wl.C, wl.Hs, wl.Ws, wl.dtype, kernel=kernel)
            self.khat = self.plan.kernel_spectrum(torch.from_numpy(wl.k).to(dev))
            self.u = up(wl.u)
            self.v = self.w = self.D = None
            self.y = torch.empty_like(self.u)
            self.outputs = wl.B * wl.C * wl.Hs * wl.Ws
        else:
            self.plan = binding.Plan(wl.B, wl.H, wl.N, wl.dtype, gated=wl.gated, kernel=kernel)
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
        if self.plan.path in ("fused", "fused_tc", "fused_umma", "fused_t2"):
            return 1
        pairs = ((self.wl.B + 1) // 2) * (self.wl.C if self.is2d else self.wl.H)
        group = max(1, self.plan.workspace_bytes // self._pair_bytes())
        return 3 * int(np.ceil(pairs / group))

    def _pair_bytes(self):
        if self.is2d:
            return self.wl.Hs * 2 * self.wl.Ws * 8
        return 2 * self.wl.N * 8

    def compute_dtype(self):
        return {"fused": "f32", "multipass": "f32", "2d": "f32", "fused_tc": "bf16", "fused_t2": "bf16",
                "fused_umma": "bf16", "2d_tc": "f32+bf16"}.get(self.plan.path, "f32")

    def dominant_kernel(self):
        return {"fused": "fused_fwd_simt", "multipass": "mp_pass2", "2d": "c2_pass2", "fused_t2": "fused_fwd_t2",
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
def workload_config(wl, path=None, world=1, shard="weak"):
    """The `config` object of a line: the workload by name and shape."""
    cfg = {"workload": wl.name, "dtype_io": wl.dtype,
           "l2": "flushed between timed steps (256 MiB write outside the events)"}
    if path:
        cfg["path"] = path
    if world > 1:
        cfg["parallelism"] = (f"channels sharded over {world} ranks, {shard} scaling, no collective on the data path")
    else:
        cfg["parallelism"] = "1 GPU"
    if hasattr(wl, "C"):
        cfg.update(B=wl.B, C=wl.C, Hs=wl.Hs, Ws=wl.Ws)
    else:
        cfg.update(B=wl.B, H=wl.H, N=wl.N, gated=wl.gated, skip_term=wl.D is not None)
    return cfg


def measure(wl, args, torch, steps, warmup, pg=None, world=1, clocks=False, e2e=True, cpu_seconds=0.0,
            config_name=None):
    """Time one workload: K device-timed steps (max over ranks), optional
    e2e, the roofline of the dominant kernel, the tensor-pipe fraction and the
    CPU oracle baseline.  Returns the result dict (the line's fields)."""
    rank = pg.get_rank() if pg else 0
    r = Runner(wl, torch, kernel=args.kernel)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    for _ in range(max(warmup, 3)):
        r.step()
    torch.cuda.synchronize()
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) if (clocks and rank == 0) else None
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
    per_step = time_steps(r, steps, torch, flush)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clk = sampler.stop() if sampler else None
    from fft_long_convolution_causal_b200.dist import max_over_ranks, sum_over_ranks
    total_ms = max_over_ranks(float(np.sum(per_step)), pg, device="cuda")
    ms_per_step = total_ms / steps
    # every rank's outputs (shards may differ by a channel) over the slowest rank's time
    job_outputs = sum_over_ranks(float(r.outputs), pg, device="cuda")
    value = job_outputs / (ms_per_step * 1e-3)

    e2e_d = None
    if e2e:
        e2e_ms, h2d, d2h = time_e2e(r, max(3, min(steps, 20)), torch)
        e2e_ms = max_over_ranks(e2e_ms, pg, device="cuda")
        e2e_d = {"value": job_outputs / (e2e_ms * 1e-3), "unit": "elems/s",
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    hbm, bf16, peak_kind = measured_peaks()
    alg_bytes = wl.io_bytes()
    # The fused paths are one launch per step, so the step's event time is that
    # kernel's time; for multi-launch paths the whole step is charged to the
    # dominant kernel (a lower bound on its achieved rate).
    achieved = alg_bytes / (ms_per_step * 1e-3) / 1e9
    kname = r.dominant_kernel()
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": recorded_traffic(config_name or wl.name, kname),
                "kernel": kname, "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": alg_bytes}
    mma = r.plan.mma_flops
    tensor = {"mma_flops_per_step": mma, "achieved_tflops": round(mma / (ms_per_step * 1e-3) / 1e12, 2),
              "peak_tflops": bf16, "peak_source": f"{peak_kind} bf16_tflops (burst)",
              "frac": round(mma / (ms_per_step * 1e-3) / 1e12 / bf16, 4)}
    cpu = None
    if cpu_seconds > 0 and rank == 0 and world == 1:
        cpu = cpu_oracle_rate(wl, cpu_seconds)
    res = {"value": value, "unit": "elems/s", "ms_per_step": ms_per_step, "steps": steps, "warmup": warmup,
           "ms_per_step_min": float(np.min(per_step)), "ms_per_step_median": float(np.median(per_step)),
           "dtype": r.compute_dtype(), "config": workload_config(wl, r.plan.path, world, args.shard),
           "roofline": roofline, "tensor_pipe": tensor, "cpu_baseline": cpu, "e2e": e2e_d,
           "gpu_launches": r.launches_per_step() * steps, "clocks": clk}
    del r
    torch.cuda.empty_cache()
    return res


def _time_fn(fn, steps, warmup, torch, flush):
    """Mean device ms of fn() over `steps` calls, L2 flushed between calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush.fill_(1)
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def variants(torch, steps=5):
    """Skipped-work variants of the long workload's shape (B=2, H=64, N=2^20,
    fp32), each timed against the dense multi-pass plan on the same inputs:
    a partial convolution (4096-tap filters, chunked on chip), a
    frequency-sparse filter (half of the outer-digit pairs dropped) and the
    state-space filters with chunked state passing (d = 16)."""
    from fft_long_convolution_causal_b200 import binding
    B, H, N = 2, 64, 1 << 20
    dev = torch.device("cuda")
    g = torch.Generator(device="cpu").manual_seed(7)
    u = torch.randn(B, H, N, generator=g).to(dev)
    D = torch.randn(H, generator=g).to(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    out = {}

    def pair(name, fn_variant, fn_dense, note):
        tv = _time_fn(fn_variant, steps, 3, torch, flush)
        td = _time_fn(fn_dense, steps, 3, torch, flush)
        out[name] = {"ms_variant": round(tv, 4), "ms_dense": round(td, 4), "speedup": round(td / tv, 3),
                     "note": note}

    dense = binding.Plan(B, H, N, "f32")
    ws = dense.new_workspace()
    y = torch.empty_like(u)
    # partial: 4096 taps
    L = 4096
    k = (torch.randn(H, L, generator=g) * torch.exp(-1e-3 * torch.arange(L, dtype=torch.float32))).to(dev)
    part = binding.PartialPlan(B, H, N, "f32", L_max=L)
    kp = part.kernel_spectrum(k)
    kd = dense.kernel_spectrum(k)
    pair("partial_l4096", lambda: part.fwd(u, kp, D=D, y=y), lambda: dense.fwd(u, kd, D=D, y=y, workspace=ws),
         "filters of 4096 taps: chunked partial plan vs the dense 2N-point multi-pass plan")
    del part, kp
    # frequency-sparse: half of the outer-digit pairs dropped (Hermitian-symmetric mask)
    kfull = (torch.randn(H, N, generator=g) * torch.exp(-1e-5 * torch.arange(N, dtype=torch.float32))).to(dev)
    sp = binding.Plan(B, H, N, "f32")
    ks = sp.kernel_spectrum(kfull)
    G = sp.spectrum_blocks
    keep = np.ones(G, bool)
    for j in range(1, G // 2 + 1):
        if j % 2 == 1:
            keep[j] = keep[(G - j) % G] = False
    sp.sparsify(ks, keep)
    kd = dense.kernel_spectrum(kfull, khat=kd)
    pair("freq_sparse_half", lambda: sp.fwd(u, ks, D=D, y=y, workspace=ws),
         lambda: dense.fwd(u, kd, D=D, y=y, workspace=ws),
         f"{int((~keep).sum())} of {G} outer-digit blocks dropped vs the same plan dense")
    del sp, ks
    # chunked state passing: d = 16 poles per channel
    d = 16
    mag = 1.0 - torch.rand(H, d, generator=g) * 1e-3
    ang = torch.rand(H, d, generator=g) * 0.1
    lam = torch.polar(mag, ang)
    c = torch.complex(torch.randn(H, d, generator=g), torch.randn(H, d, generator=g)) * 0.1
    ssm = binding.SSMPlan(B, H, N, "f32", d_state=d, chunk=8192)
    kss = ssm.set_filters(lam, c)
    tt = torch.arange(N, dtype=torch.float64, device=dev)
    kmat = torch.zeros(H, N, dtype=torch.float64, device=dev)
    lam64, c64 = lam.to(torch.complex128).to(dev), c.to(torch.complex128).to(dev)
    for j in range(d):  # the same filters materialised (fp64) for the dense plan
        kmat += (c64[:, j:j + 1] * torch.exp(tt[None, :] * torch.log(lam64[:, j:j + 1]))).real
    kmat_f32 = kmat.to(torch.float32)
    kd = dense.kernel_spectrum(kmat_f32, khat=kd)
    del kmat, tt
    pair("ssm_chunked_d16", lambda: ssm.fwd(u, kss, D=D, y=y), lambda: dense.fwd(u, kd, D=D, y=y, workspace=ws),
         "diagonal state-space filters, chunks of 8192 with the state passed vs the dense plan on the same filters")
    # the same filters in bf16: chunks of 4096 on the two-stage tensor-core kernel,
    # against the bf16 dense multi-pass plan
    ub = u.to(torch.bfloat16)
    yb = torch.empty_like(ub)
    ssmb = binding.SSMPlan(B, H, N, "bf16", d_state=d, chunk=4096)
    kssb = ssmb.set_filters(lam, c)
    denseb = binding.Plan(B, H, N, "bf16")
    wsb = denseb.new_workspace()
    kdb = denseb.kernel_spectrum(kmat_f32)
    pair("ssm_chunked_d16_bf16", lambda: ssmb.fwd(ub, kssb, D=D, y=yb),
         lambda: denseb.fwd(ub, kdb, D=D, y=yb, workspace=wsb),
         "bf16: chunks of 4096 on the two-stage tensor-core kernel with the state passed vs the bf16 dense plan")
    del ssmb, kssb, denseb, wsb, kdb, ub, yb, kmat_f32
    del ssm, kss, dense, ws, u, y
    torch.cuda.empty_cache()
    # the backward pass on the Hyena-style layer (B=8, H=768, N=4096 bf16): du through the
    # forward kernel with the conjugated spectrum, then dk and dD; against the forward
    Bh, Hh, Nh = 8, 768, 4096
    plan = binding.Plan(Bh, Hh, Nh, "bf16")
    kh = (torch.randn(Hh, Nh, generator=g) * torch.exp(-1e-3 * torch.arange(Nh, dtype=torch.float32))).to(dev)
    khat = plan.kernel_spectrum(kh)
    kconj = plan.spectrum_conjugate(khat)
    uh = torch.randn(Bh, Hh, Nh, generator=g).to(dev, torch.bfloat16)
    dyh = torch.randn(Bh, Hh, Nh, generator=g).to(dev, torch.bfloat16)
    Dh = torch.randn(Hh, generator=g).to(dev)
    yh = torch.empty_like(uh)
    tb = _time_fn(lambda: plan.bwd(dyh, uh, khat, kconj, D=Dh), steps, 3, torch, flush)
    tf = _time_fn(lambda: plan.fwd(uh, khat, D=Dh, y=yh), steps, 3, torch, flush)
    out["backward_hyena"] = {"ms_backward": round(tb, 4), "ms_forward": round(tf, 4),
                             "ratio": round(tb / tf, 3), "path": plan.path,
                             "note": "du, dk, dD of the Hyena-style layer against its forward"}
    del plan, khat, kconj, uh, dyh, yh
    torch.cuda.empty_cache()
    # the 3-D causal convolution (no named workload is 3-D): B=2, C=8, 64^3 fp32
    # volumes with full-size filters; output elements per second and the HBM
    # fraction of u + y
    B3, C3, S3 = 2, 8, 64
    plan = binding.Plan3D(B3, C3, S3, S3, S3, "f32")
    k3 = torch.randn(C3, S3, S3, S3, generator=g).to(dev)
    kh3 = plan.kernel_spectrum(k3)
    u3 = torch.randn(B3, C3, S3, S3, S3, generator=g).to(dev)
    y3 = torch.empty_like(u3)
    ws3 = plan.new_workspace()
    t3 = _time_fn(lambda: plan.fwd(u3, kh3, y=y3, workspace=ws3), steps, 3, torch, flush)
    n3 = B3 * C3 * S3 ** 3
    hbm, _, _ = measured_peaks()
    out["conv3d_b2_c8_64cubed_f32"] = {"ms": round(t3, 4), "elems_per_s": n3 / (t3 * 1e-3),
                                      "hbm_frac": round(2 * n3 * 4 / (t3 * 1e-3) / 1e9 / hbm, 4), "path": plan.path,
                                      "note": "five launches per group (rows, columns, depth with the product, "
                                              "inverse columns, inverse rows) through an fp32 workspace"}
    del plan, kh3, u3, y3, ws3, k3
    torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args.record_traffic, args.config, args.channels, args.traffic_command)
        return 0
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
    wl = build_workload(args.config, args.channels, rank, world, args.shard)
    head = measure(wl, args, torch, args.steps, args.warmup, pg=pg, world=world, clocks=not args.no_clocks,
                   e2e=not args.no_e2e, cpu_seconds=0.0 if args.no_cpu_baseline else args.cpu_seconds,
                   config_name=args.config)
    del wl
    per_config = None
    if world == 1 and not args.no_per_config and not args.channels:
        from fft_long_convolution_causal_b200 import workloads
        per_config = {}
        for name in workloads.CONFIG_ORDER:
            if name == args.config:
                continue
            w2 = build_workload(name)
            res = measure(w2, args, torch, args.per_config_steps, 3, clocks=False, e2e=not args.no_e2e,
                          cpu_seconds=0.0 if args.no_cpu_baseline else min(args.cpu_seconds, 5.0),
                          config_name=name)
            del w2
            per_config[name] = res
    var = None
    if world == 1 and not args.no_variants and not args.channels:
        var = variants(torch)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": head["value"], "unit": "elems/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak" if (world == 1 or args.shard == "weak") else "strong", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic", "config": head["config"],
            "roofline": head["roofline"], "tensor_pipe": head["tensor_pipe"], "cpu_baseline": head["cpu_baseline"],
            "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
            "ms_per_step_min": head["ms_per_step_min"], "ms_per_step_median": head["ms_per_step_median"]}
    if per_config is not None:
        line["per_config"] = per_config
    if var is not None:
        line["variants"] = var
    print(json.dumps(line))
    return 0


def main_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 times it on the host cores, each
    step a bounded uniform sample of the workload's outputs."""
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
    cfg = workload_config(wl, "oracle (CPU fp64 direct sum)", 1, args.shard)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "elems/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(times)) * 1e3,
            "outputs_per_step": n, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": value, "unit": "elems/s", "cores": s.oracle.num_threads(), "kind": "oracle",
                             "sample": "each step: " + s.describe(n, float(np.mean(times)))},
            "e2e": {"value": value, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
