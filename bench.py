"""Benchmark of the TARA-biased joint attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload full] [--impl ours|reference]

One step = one call of tara_attn_forward (tile summaries + the attention kernel) over the
workload's whole batch, inputs resident in HBM.  The default workload is the 56-head,
107,126-token bf16 shot with reference binding (Q/K/V/O 6.1 GB, far above the 126 MB L2, so
no L2 flush is needed between steps).  With --gpus N > 1 (torchrun), every rank runs its own
replica of the workload with no collective on the data path (weak scaling); the time is the
max over ranks.  Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle instead, on bounded row samples of the same
workload (the pages ship no code to run, so the oracle is the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_dram_traffic.txt")
CSRC = os.path.join(ROOT, "video_diffusion_attention_b200", "csrc")


def describe(w: W.Workload) -> dict:
    segs = []
    names = {0: "text", 1: "picture", 2: "target", 3: "guide", 4: "audio", 5: "other_video"}
    for s in w.segments:
        d = {"role": names[s.kind], "tokens": s.length}
        if s.frames > 1:
            d["frames"] = s.frames
        segs.append(d)
    return {"workload": "%s: B=%d H=%d N=%d D=%d %s" % (w.name, w.B, w.H, w.N, w.D, w.dtype),
            "B": w.B, "H": w.H, "N": w.N, "head_dim": w.D, "segments": segs,
            "params": {"window": w.params.window, "falloff": w.params.falloff,
                       "strength": w.params.strength, "cap": w.params.cap,
                       "gain": list(w.params.gain)},
            "flop_per_step": w.flops,
            "l2": "inputs %.1f GB > 126 MB L2; no flush" % (4 * w.B * w.H * w.N * w.D * 2 / 1e9)}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# the device sources each attention kernel is compiled from (the tile-summary kernel lays out
# the records both read; the quantiser the 8-bit codes the INT8 kernel reads)
KERNEL_SOURCES = ("attn_pair.cuh", "attn_tc.cuh", "sm100_ptx.cuh", "tara_common.cuh",
                  "tile_summary.cuh")
KERNEL_SOURCES_INT8 = ("attn_tc.cuh", "quant_int8.cuh", "sm100_ptx.cuh", "tara_common.cuh",
                       "tile_summary.cuh")


def kernel_source_hash(sources=KERNEL_SOURCES) -> str:
    """sha256 (first 16 hex digits) of a kernel's device sources with // comments, trailing
    blanks and empty lines removed: edits to comments leave it unchanged, edits to code do not."""
    import re
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(CSRC, f)) as fh:
            lines = (re.sub(r"//.*$", "", line).rstrip() for line in fh.read().splitlines())
            code = "\n".join(line for line in lines if line)
        h.update(f.encode() + code.encode())
    return h.hexdigest()[:16]


def clock_normalised(achieved: float, peak: float, kernel_mhz, peaks: dict) -> dict:
    """The roofline fraction with the peak moved to the kernel's own SM clock.

    The sustained peak was measured at the clock a dense GEMM settles at under the power cap;
    a kernel that leaves the tensor pipe idle part of the time runs at a higher clock, which
    flatters achieved/peak.  Scaling the peak by kernel MHz / peak MHz compares work per clock
    cycle instead (the figure ncu's tensor-pipe-active counter reads).  None when either clock
    is unknown."""
    peak_mhz = (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")
    if not kernel_mhz or not peak_mhz:
        return {"frac_at_kernel_clock": None, "kernel_sm_mhz_median": kernel_mhz,
                "peak_sm_mhz_median": peak_mhz}
    peak_at_clock = peak * float(kernel_mhz) / float(peak_mhz)
    return {"frac_at_kernel_clock": achieved / peak_at_clock,
            "peak_at_kernel_clock": peak_at_clock,
            "kernel_sm_mhz_median": kernel_mhz, "peak_sm_mhz_median": peak_mhz}


def measure_int8_gemm_tops(dev, n: int = 8192, seconds: float = 2.0):
    """Dense int8 GEMM rate of this GPU (TOPS, 2*n^3 per product) through torch._int_mm:
    best of 10 single products (burst), the mean over products run back to back for about
    `seconds` (sustained, at the clock a long dense contraction settles at under the power
    cap) and that clock (median SM MHz sampled meanwhile).  Nones if the call is unavailable."""
    import torch
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize(dev)
    except (RuntimeError, AttributeError):
        return None, None, None
    ops = 2.0 * n ** 3
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize(dev)
        best = min(best, e0.elapsed_time(e1))
    reps = max(10, int(seconds * 1e3 / best))
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        torch._int_mm(a, b)
    e1.record()
    torch.cuda.synchronize(dev)
    clk = sampler.stop()
    sustained_ms = e0.elapsed_time(e1) / reps
    return ops / (best * 1e-3) / 1e12, ops / (sustained_ms * 1e-3) / 1e12, clk.get("sm_mhz")


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it was
    taken on the current kernel source; None otherwise."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    vals = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if "=" in line:
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    # "<workload>_int8" figures belong to the INT8 kernel, the others to the 16-bit one; each
    # kernel's figures carry the hash of its sources (kernel_source_sha256_16[_int8]), and a
    # figure may carry its own (taken on an earlier version of the same kernel)
    key = "bytes_per_launch_" + workload
    int8 = workload.endswith("_int8")
    default = vals.get("kernel_source_sha256_16_int8" if int8 else "kernel_source_sha256_16")
    current = kernel_source_hash(KERNEL_SOURCES_INT8 if int8 else KERNEL_SOURCES)
    if vals.get("kernel_source_sha256_16_" + workload, default) != current:
        return None
    return float(vals[key]) if key in vals else None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            import torch
            p = torch.cuda.get_device_properties(self.device_index)
            bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", bus, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        under_load = [x for x in sm if x > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(under_load) if under_load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample_rate(w: W.Workload, budget_s: float, device_inputs=None, seed: int = 11):
    """Time the oracle on seeded query rows of workload w for about budget_s seconds.

    Returns (rows, seconds, threads).  Inputs are the workload's own seeded tensors (drawn on
    the GPU when one is given, else on the CPU)."""
    import torch
    import oracle
    if device_inputs is not None:
        q, k, v = device_inputs
    else:
        q, k, v = W.make_qkv(w, "cpu")
    raw = [oracle.torch_to_numpy_raw(t) for t in (q, k, v)]
    meta = oracle.pack_token_meta(w.segments)
    rng = np.random.Generator(np.random.PCG64(seed))
    threads = oracle.max_threads()

    def run(n):
        rows = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.H, n),
                         rng.integers(0, w.N, n)], axis=1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention_rows(raw[0][0], raw[1][0], raw[2][0], raw[0][1], meta, w.params, rows)
        return time.perf_counter() - t0

    probe = max(threads, 16)
    dt = run(probe)
    n = max(probe, int(probe * budget_s / max(dt, 1e-6)))
    dt = run(n)
    return n, dt, threads


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def run_reference(args, w: W.Workload):
    """The oracle arm: K timed steps, each a bounded row sample of the workload."""
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v = W.make_qkv(w, "cpu")
    raw = [oracle.torch_to_numpy_raw(t) for t in (q, k, v)]
    meta = oracle.pack_token_meta(w.segments)
    threads = oracle.max_threads()
    rng = np.random.Generator(np.random.PCG64(5))
    flop_per_row = 4.0 * w.N * w.D
    # size one step at about 8 s of CPU work
    probe = max(16, threads)
    rows = np.stack([rng.integers(0, w.B, probe), rng.integers(0, w.H, probe),
                     rng.integers(0, w.N, probe)], axis=1).astype(np.int64)
    t0 = time.perf_counter()
    oracle.attention_rows(raw[0][0], raw[1][0], raw[2][0], raw[0][1], meta, w.params, rows)
    per_row = (time.perf_counter() - t0) / probe
    n = max(threads, int(8.0 / max(per_row, 1e-9)))
    times = []
    for step in range(args.warmup + args.steps):
        rows = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.H, n),
                         rng.integers(0, w.N, n)], axis=1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention_rows(raw[0][0], raw[1][0], raw[2][0], raw[0][1], meta, w.params, rows)
        if step >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = n * len(times) * flop_per_row / total / 1e12
    sample = "%d random query rows per step of %s (each row: all %d keys, fp64)" % (n, w.name, w.N)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": describe(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


METRIC = "biased-attn fwd TFLOP/s at 107,126 tok bf16; % of B200 dense-BF16 peak"


def max_over_ranks(values, device="cpu"):
    """Element-wise max of a list of timings over all ranks of the default process group
    (the slowest rank defines a multi-GPU time); identity without a group."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(flop_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own replica (weak scaling), so the job does
    world * flop_per_rank per step in the slowest rank's step time."""
    return world * flop_per_rank / (ms_per_step * 1e-3) / 1e12


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="full", choices=W.ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    w = W.get(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    import torch
    import torch.distributed as dist
    import video_diffusion_attention_b200 as T

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    lib = T.load_library()   # raises if the CUDA library is missing: no fallback
    q, k, v = W.make_qkv(w, dev)
    meta = T.DeviceMeta(T.pack_token_meta(w.segments), dev)
    params = T.params_from(w.params)
    O = torch.empty_like(q)
    L = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        T.attn_forward(q, k, v, meta, params, O, L, stream)
    torch.cuda.synchronize(dev)
    if T.device_status() != 0:
        raise SystemExit("kernel reported a device timeout during warm-up")

    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in kev:   # create the events' handles; the library re-records them per call
        a.record(stream)
        b.record(stream)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(args.steps):
        T.set_kernel_events(*kev[i])
        T.attn_forward(q, k, v, meta, params, O, L, stream)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    if T.device_status() != 0:
        raise SystemExit("kernel reported a device timeout in the timed region")
    ms_total = start.elapsed_time(stop)
    kernel_ms = [a.elapsed_time(b) for a, b in kev]
    kernel_ms_median = statistics.median(kernel_ms)
    ms_total, kmean = max_over_ranks([ms_total, statistics.mean(kernel_ms)], dev)
    ms_step = ms_total / args.steps
    value = job_throughput(w.flops, world, ms_step)

    # end to end through the C ABI with host buffers (tara_attn_forward_host): every step
    # copies Q/K/V and the metadata in from pinned host memory and O/LSE back out, all inside
    # the timed region; the library pipelines the copies against the kernels chunk by chunk
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hmeta = T.HostMeta({key: getattr(meta, key).cpu().numpy() for key in ("seg", "time_s", "pic", "m")})
    hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    hL = torch.empty(L.shape, dtype=L.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv)) + sum(
        getattr(hmeta, key).numel() * getattr(hmeta, key).element_size()
        for key in ("seg", "time_s", "pic", "m"))
    d2h = hO.numel() * hO.element_size() + hL.numel() * hL.element_size()

    def e2e_step():
        T.attn_forward_host(hq, hk, hv, hmeta, params, hO, hL, stream)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / args.e2e_steps], dev)[0]
    e2e_value = job_throughput(w.flops, world, e2e_ms)

    # the step before the path, measured on its own: pixel mask of a prepared 107-frame shot at
    # 544x928 (the resolution of the pages' user run) to the workload's 26-frame target grid
    mask_line = None
    tgt = [sg for sg in w.segments if sg.kind == W.TARGET]
    if tgt and tgt[0].tokens_per_frame == 2000:
        px = torch.from_numpy(W.pixel_ellipse_mask(w.seed(3) + 1, 107, 544, 928)).to(dev)
        mo = torch.empty((tgt[0].frames, 40, 50), dtype=torch.float32, device=dev)
        for _ in range(3):
            T.prepare_target_mask(px, 107, 4, tgt[0].frames, 40, 50, out=mo, stream=stream)
        # one event pair around each launch: a ~45 us kernel is shorter than the Python call
        # that launches it, so events around a back-to-back loop would time the host instead
        reps = 20
        mev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize(dev)
        for a, b in mev:
            a.record(stream)
            T.prepare_target_mask(px, 107, 4, tgt[0].frames, 40, 50, out=mo, stream=stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
        mms = statistics.median(a.elapsed_time(b) for a, b in mev)
        mbytes = px.numel() * 4 + mo.numel() * 4
        mask_line = {"kernel": "target_mask_narrow_kernel (rows <= 1024 px)", "workload": "107x544x928 fp32 pixel mask -> "
                     "%dx40x50 target weights" % tgt[0].frames, "ms": mms, "bound": "hbm",
                     "algorithmic_bytes": mbytes, "achieved_GBs": mbytes / (mms * 1e-3) / 1e9}
    # the INT8 Q K^T variant of the same forward (Q per token, K per 128-key block, 8-bit
    # tensor cores for Q K^T, P V in bf16): reported beside the headline, never as it
    q8_line = None
    if w.D == 128 and w.dtype in ("bf16", "fp16"):
        p8 = T.params_from(w.params, qk_int8=1)
        for _ in range(2):
            T.attn_forward(q, k, v, meta, p8, O, L, stream)
        reps = 5
        kev8 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(reps)]
        for a, b in kev8:
            a.record(stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(reps):
            T.set_kernel_events(*kev8[i])
            T.attn_forward(q, k, v, meta, p8, O, L, stream)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        if T.device_status() != 0:
            raise SystemExit("INT8 kernel reported a device timeout")
        q8_step = s0.elapsed_time(s1) / reps
        q8_kernel = statistics.mean(a.elapsed_time(b) for a, b in kev8)
        q8_line = {"kernel": "attn_tc_kernel<int8 QK>", "ms_per_step": q8_step,
                   "value": w.flops / (q8_step * 1e-3) / 1e12, "unit": "TFLOP/s",
                   "kernel_ms": q8_kernel, "flop_basis": "4*B*H*N^2*D, as the headline",
                   "gpu_launches_per_step": 4}
    peaks, peak_src = load_peaks()
    if q8_line is not None:
        # QK^T (half the FLOP) at the int8 GEMM rate measured here, PV at the bf16 peak
        p16 = float(peaks["bf16_tflops_sustained"])
        p8_burst, p8, p8_mhz = measure_int8_gemm_tops(dev)
        if p8 is not None:
            p8_kind = ("QK^T at the dense int8 GEMM rate measured in this run (torch._int_mm "
                       "8192^3 back to back for 2 s: %.0f TOPS; best single product %.0f TOPS), "
                       "PV at measured sustained bf16 (%s)" % (p8, p8_burst, peak_src))
        else:
            p8 = 2.0 * p16
            p8_kind = ("QK^T at 2 x measured sustained bf16 (nominal int8 ratio; the int8 GEMM "
                       "could not be timed), PV at measured sustained bf16 (%s)" % peak_src)
        q8_peak = 1.0 / (0.5 / p8 + 0.5 / p16)
        q8_ach = w.flops / (q8_line["kernel_ms"] * 1e-3) / 1e12
        q8_line["roofline"] = {"bound": "tensor", "achieved": q8_ach, "peak": q8_peak,
                               "unit": "TFLOP/s", "frac": q8_ach / q8_peak,
                               "traffic": recorded_traffic(w.name + "_int8"),
                               "int8_tops_sustained": p8, "int8_tops_burst": p8_burst,
                               "peak_kind": p8_kind}
        # per clock: each half's peak moved to the kernel's clock from the clock it was
        # measured at (the int8 GEMM's sampled here, the bf16 GEMM's from the peaks file)
        kmhz = clk.get("sm_mhz")
        p16_mhz = (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")
        if kmhz and p16_mhz and p8_mhz:
            pk = 1.0 / (0.5 / (p8 * kmhz / p8_mhz) + 0.5 / (p16 * kmhz / p16_mhz))
            q8_line["roofline"]["clock_normalised"] = {
                "frac_at_kernel_clock": q8_ach / pk, "peak_at_kernel_clock": pk,
                "kernel_sm_mhz_median": kmhz, "int8_peak_sm_mhz_median": p8_mhz,
                "bf16_peak_sm_mhz_median": p16_mhz}
        else:
            q8_line["roofline"]["clock_normalised"] = {"frac_at_kernel_clock": None}
    if mask_line is not None:
        mask_line["peak_GBs"] = float(peaks["hbm_gbs"])
        mask_line["frac"] = mask_line["achieved_GBs"] / float(peaks["hbm_gbs"])
    achieved = w.flops / (kmean * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops_sustained"])
    traffic = recorded_traffic(w.name)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Q/K/V ~ N(0,1), packed shot layout; no dataset or weights)",
        "config": describe(w),
        "pct_of_dense_bf16_peak": {
            "sustained_measured": 100.0 * value / world / float(peaks["bf16_tflops_sustained"]),
            "burst_measured": 100.0 * value / world / float(peaks["bf16_tflops"]),
            "nominal_2250": 100.0 * value / world / 2250.0, "peaks_source": peak_src},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "attn_pair_kernel", "kernel_ms": kmean,
                     "clock_normalised": clock_normalised(achieved, peak, clk.get("sm_mhz"), peaks),
                     "kernel_ms_median": kernel_ms_median,
                     "peak_kind": "bf16_tflops_sustained (%s): the kernel runs back to back for "
                                  "seconds" % peak_src},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    if mask_line is not None:
        line["mask_prep"] = mask_line
    if q8_line is not None:
        line["int8_qk"] = q8_line
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, dt, threads = oracle_sample_rate(w, args.cpu_budget, device_inputs=(q, k, v))
        line["cpu_baseline"] = {
            "value": n * 4.0 * w.N * w.D / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": "%d seeded query rows of %s in %.1f s (each row against all %d keys, "
                      "fp64)" % (n, w.name, dt, w.N),
            "extrapolated_full_call_s": dt / n * w.B * w.H * w.N}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
