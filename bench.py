"""Benchmark: one step = the whole hot path (forward O/LSE, then backward:
rowsum preprocess, main backward, dQ conversion) over one batch of synthetic
input already resident in HBM.

Metric: attention TFLOP/s counting only allowed (unmasked) score entries,
4*D per pair forward and 10*D per pair backward, and the fraction of the B200
dense 16-bit tensor peak.  Default workload: LTX diffusion shape, bf16,
B=1, H=32, Sq=Sk=15300, D=128, no mask.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

One process per GPU (torchrun for N > 1): every rank runs the same workload on
its own GPU (the attention units are independent; there is no exchange), the
step time is the max over ranks and the value is the work of all ranks over
that time (weak scaling).  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
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

import torch  # noqa: E402

from scaled_dot_product_12_b200 import synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_DENSE_BF16_TFLOPS = 2250.0  # NVIDIA B200 dense fp16/bf16 (the 2:4-sparse figure halved)
CLOCK_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing (no data-path collective: only barrier + max of times)
# ---------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clocks not sampled"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 5:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]),
                                 int(parts[4], 16) if parts[4].startswith("0x") else int(parts[4])))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for bit, name in CLOCK_REASONS.items():
                if r[3] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": sorted(reasons),
                "samples": len(loaded), "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------
def workload_flops(w: synth.Workload):
    from scaled_dot_product_12_b200 import binding as B
    pairs = B.allowed_pairs(w.Sq, w.Sk, w.window_left, w.window_right, w.bottom_right)
    n = pairs * w.B * w.H
    return 4 * w.D * n, 10 * w.D * n, n


def describe(w: synth.Workload):
    return {"workload": f"{w.name}: {w.describe}, fwd+bwd", "B": w.B, "H": w.H, "Sq": w.Sq,
            "Sk": w.Sk, "D": w.D, "dtype": w.dtype,
            "window": [w.window_left, w.window_right], "layout": "BHSD dense, LSE HT",
            "l2": "inputs larger than L2 (Q, K, V, O, dO, dQ, dK, dV each "
                  f"{w.B * w.H * w.Sq * w.D * 2 / 1e6:.0f} MB; L2 is 126 MB)"}


class Step:
    """Device buffers and the two C-ABI calls of one step."""

    def __init__(self, w: synth.Workload, dev):
        from scaled_dot_product_12_b200 import binding as B
        self.B = B
        self.w = w
        dtype = synth.DTYPES[w.dtype]
        q, k, v, do = synth.qkv_do((w.B, w.H, w.Sq, w.D), (w.B, w.H, w.Sk, w.D), w.seed, dtype)
        self.host = {"q": q, "k": k, "v": v, "do": do}
        self.q, self.k, self.v, self.do = (t.to(dev) for t in (q, k, v, do))
        self.scale = w.D ** -0.5
        self.window = (w.window_left, w.window_right)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
        self.dq = torch.empty_like(self.q)
        self.dk = torch.empty_like(self.k)
        self.dv = torch.empty_like(self.v)
        pr = B.Problem(self.q, self.k, self.scale, self.window, w.bottom_right, None, None, None,
                       None, "HT")
        self.bp = B.bwd_params(self.do, self.q, self.k, self.v, self.o, self.lse, pr, self.dq,
                               self.dk, self.dv)
        self.ws = torch.empty(max(1, B.workspace_bytes(self.bp)), dtype=torch.uint8, device=dev)
        self.bp.workspace = self.ws.data_ptr()
        self.bp.workspace_bytes = self.ws.numel()

    def run(self, stream, ev=None):
        """ev: optional list of 4 events: fwd start/end, bwd-main start/end."""
        import ctypes
        B = self.B
        if ev is not None:
            ev[0].record(stream)
        B.forward(self.q, self.k, self.v, sm_scale=self.scale, window=self.window,
                  bottom_right=self.w.bottom_right, out=self.o, lse=self.lse, stream=stream)
        if ev is not None:
            ev[1].record(stream)
            self.bp.main_kernel_events[0] = ev[2].cuda_event
            self.bp.main_kernel_events[1] = ev[3].cuda_event
        else:
            self.bp.main_kernel_events[0] = None
            self.bp.main_kernel_events[1] = None
        B._check("attn_bwd", B.lib().attn_bwd(ctypes.byref(self.bp), stream.cuda_stream))


def run_gpu(args, rank, world, local):
    from scaled_dot_product_12_b200 import binding as B
    w = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    step = Step(w, dev)
    stream = torch.cuda.Stream(dev)
    fwd_flops, bwd_flops, pairs = workload_flops(w)
    flops = fwd_flops + bwd_flops
    peaks, peak_src = load_peaks()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step.run(stream)
    stream.synchronize()
    if B.device_status(dev, stream) != 0:
        raise RuntimeError("a device-side wait gave up during warm-up")

    # ---- device-timed region: K steps, inputs resident in HBM ----
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for evs in events:  # torch creates an event on its first record: make the handles exist
        for e in evs:
            e.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(args.steps):
                step.run(stream, events[i])
            t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms_total = t0.elapsed_time(t1)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in events) / args.steps
    main_ms = sum(e[2].elapsed_time(e[3]) for e in events) / args.steps
    status = B.device_status(dev, stream)
    if status != 0:
        raise RuntimeError(f"a device-side wait gave up (status {status:#x})")
    clock_summary = clocks.summary()

    total_flops = sum_over_ranks(flops, world)
    value = total_flops / (ms_step * 1e-3) / 1e12
    # The denominator follows the clocks seen in the timed region: the burst
    # GEMM figure while the SM clock stayed at its maximum, the sustained
    # (power-capped) one once the power cap lowered it.  Both fractions are
    # reported.
    burst = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    capped = power_capped(clock_summary)
    peak = sustained if capped else burst
    fwd_tf = fwd_flops / (fwd_ms * 1e-3) / 1e12
    bwd_tf = bwd_flops / (main_ms * 1e-3) / 1e12
    dominant = ("attn_bwd_kernel", bwd_tf, main_ms) if main_ms >= fwd_ms else ("attn_fwd_kernel",
                                                                              fwd_tf, fwd_ms)
    traffic = load_traffic(dominant[0], w.name)

    # ---- end to end through the C ABI with host buffers ----
    e2e = run_e2e(step, stream, dev, min(args.steps, 5), flops, world)

    line = {
        "metric": "attention TFLOP/s (fwd+bwd, unmasked FLOPs)", "value": round(value, 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp16",
        "data": "synthetic: i.i.d. N(0,1) Q, K, V, dO from a fixed seed",
        "config": describe(w),
        "fwd": {"ms": round(fwd_ms, 4), "tflops": round(fwd_tf, 1),
                "frac_of_peak": round(fwd_tf / peak, 4),
                "frac_of_burst": round(fwd_tf / burst, 4)},
        "bwd_main": {"ms": round(main_ms, 4), "tflops": round(bwd_tf, 1),
                     "frac_of_peak": round(bwd_tf / peak, 4),
                     "frac_of_burst": round(bwd_tf / burst, 4)},
        "bwd_other_ms": round(ms_step - fwd_ms - main_ms, 4),
        # The delta preprocess and the dQ conversion are HBM-bound: their
        # algorithmic bytes over the rest of the step (both kernels and the
        # gaps between launches) give a lower bound on their bandwidth.
        "bwd_other": other_bandwidth(w, world, ms_step - fwd_ms - main_ms,
                                     peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])),
        "frac_of_peak": {"measured_burst": round(value / world / burst, 4),
                         "measured_sustained": round(value / world / sustained, 4),
                         "datasheet_dense": round(value / world / DATASHEET_DENSE_BF16_TFLOPS, 4)},
        "roofline": {"bound": "tensor", "kernel": dominant[0], "achieved": round(dominant[1], 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(dominant[1] / peak, 4),
                     "peak_source": (f"{peak_src} bf16_tflops_sustained (the power cap "
                                     "lowered the SM clock in the timed region)") if capped else
                                    (f"{peak_src} bf16_tflops (burst: the SM clock stayed at "
                                     "its maximum during the timed region)"),
                     "traffic": traffic},
        "gpu_launches": 4 * args.steps,
        "clocks": clock_summary,
        "e2e": e2e,
        "allowed_pairs": pairs,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def other_bandwidth(w, world, ms, hbm_gbs):
    """Preprocess reads O, dO (2 x 2D bytes per row and head) and writes delta
    (4) and the zeroed fp32 dQ accumulator (4D); the conversion reads the
    accumulator (4D) and writes dQ (2D): (14 D + 4) bytes per row and head."""
    rows = w.B * w.Sq * w.H  # the bench workloads are dense
    nbytes = rows * (14 * w.D + 4) * world
    gbs = nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None
    return {"ms": round(ms, 4), "bytes": nbytes, "gbs": round(gbs, 1) if gbs else None,
            "peak_gbs": hbm_gbs, "frac": round(gbs / hbm_gbs, 4) if gbs else None}


def power_capped(clocks):
    """True if the power cap actually lowered the SM clock during the timed
    region: a median SM clock more than 3 % under the maximum.  A cap flag
    alone, with the clock still at its maximum, leaves the burst figure the
    right denominator."""
    mhz, top = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    return bool(mhz and top and mhz < 0.97 * top)


KERNEL_SOURCES = ("common.cuh", "mask.cuh", "fwd.h", "fwd.cu", "bwd.cu")


def kernels_sha256():
    """Hash of the kernel sources, to tie committed counters to a kernel build."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "scaled_dot_product_12_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def load_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if one
    for this kernel and workload exists and was taken on the kernel sources
    built now (else null: counters of another build do not describe this one)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernels_sha256") != kernels_sha256():
        return None
    return d.get("bytes_per_launch", {}).get(f"{kernel}:{workload}")


def run_e2e(step: Step, stream, dev, n, flops, world):
    """The same step through the C ABI with pinned HOST inputs and outputs: H2D
    of Q, K, V, dO and D2H of O, LSE, dQ, dK, dV inside the timed region."""
    host_in = {k: v.pin_memory() for k, v in step.host.items()}
    outs = ["o", "lse", "dq", "dk", "dv"]
    host_out = {k: torch.empty(getattr(step, k).shape, dtype=getattr(step, k).dtype,
                               pin_memory=True) for k in outs}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(n):
            step.q.copy_(host_in["q"], non_blocking=True)
            step.k.copy_(host_in["k"], non_blocking=True)
            step.v.copy_(host_in["v"], non_blocking=True)
            step.do.copy_(host_in["do"], non_blocking=True)
            step.run(stream)
            for k in outs:
                host_out[k].copy_(getattr(step, k), non_blocking=True)
        t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1) / n, world)
    total = sum_over_ranks(flops, world)
    return {"value": round(total / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


# ---------------------------------------------------------------------------
# the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def oracle_sample(w: synth.Workload, rows: int):
    """Inputs of a bounded sample: head (0, 0), the first `rows` query rows
    (all rows if rows <= 0) against all keys, and its FLOP count."""
    import numpy as np
    dtype = synth.DTYPES[w.dtype]
    q, k, v, do = synth.qkv_do((w.B, w.H, w.Sq, w.D), (w.B, w.H, w.Sk, w.D), w.seed, dtype)
    f = lambda t: t[0, 0].float().numpy().astype(np.float64)  # noqa: E731
    qn, kn, vn, don = f(q), f(k), f(v), f(do)
    if rows > 0:
        qn, don = qn[:rows], don[:rows]
    from scaled_dot_product_12_b200 import binding as B
    pairs = B.allowed_pairs(qn.shape[0], w.Sk, w.window_left, w.window_right, w.bottom_right) \
        if rows <= 0 or w.window_left == synth.WINDOW_INF and w.window_right == synth.WINDOW_INF \
        else None
    if pairs is None:
        from oracle import attn_ref as ref
        m = ref.allowed(w.Sq, w.Sk, w.window_left, w.window_right, w.bottom_right,
                        rows=list(range(qn.shape[0])))
        pairs = int(m.sum())
    return (qn, kn, vn, don), 14 * w.D * pairs


def oracle_step(w, inputs):
    """One oracle forward and backward; returns their wall times (s)."""
    from oracle import attn_ref as ref
    qn, kn, vn, don = inputs
    # rows of a prefix keep their own mask only when the window does not
    # depend on seqlen_q; the default workloads are unmasked or top-left.
    t0 = time.perf_counter()
    ref.forward(qn, kn, vn, w.D ** -0.5, w.window_left, w.window_right, w.bottom_right)
    t1 = time.perf_counter()
    ref.backward(qn, kn, vn, don, w.D ** -0.5, w.window_left, w.window_right, w.bottom_right)
    return t1 - t0, time.perf_counter() - t1


def cpu_baseline(w: synth.Workload, rows: int = 0):
    inputs, flops = oracle_sample(w, rows)
    t_f, t_b = oracle_step(w, inputs)
    dt = t_f + t_b
    pair_flops = flops / (14 * w.D)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _blas_threads(),
            "kind": "oracle", "cpu_count": os.cpu_count(),
            "fwd_tflops": round(4 * w.D * pair_flops / t_f / 1e12, 6),
            "bwd_tflops": round(10 * w.D * pair_flops / t_b / 1e12, 6),
            "sample": f"fp64 NumPy oracle, forward + backward of head (0,0) "
                      f"({'all' if rows <= 0 else rows} query rows x {w.Sk} keys, "
                      f"{flops / 1e9:.1f} GFLOP at 14*D per pair), {dt:.1f} s on "
                      f"{os.cpu_count()} host cores"}


def run_reference(args, rank, world):
    """--impl reference: the oracle as it stands, timed on the host cores."""
    w = synth.WORKLOADS[args.workload]
    rows = 256
    inputs, flops = oracle_sample(w, rows)
    for _ in range(args.warmup):
        oracle_step(w, inputs)
    t = time.perf_counter()
    t_f = t_b = 0.0
    for _ in range(args.steps):
        f_s, b_s = oracle_step(w, inputs)
        t_f, t_b = t_f + f_s, t_b + b_s
    dt = (time.perf_counter() - t) / args.steps
    pair_flops = flops / (14 * w.D)
    value = flops / dt / 1e12
    sample = (f"each step: fp64 NumPy oracle forward + backward of head (0,0), first {rows} "
              f"query rows against all {w.Sk} keys ({flops / 1e9:.2f} GFLOP)")
    return {"impl": "reference", "metric": "attention TFLOP/s (fwd+bwd, unmasked FLOPs)",
            "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": describe(w),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _blas_threads(),
                             "kind": "oracle", "sample": sample, "cpu_count": os.cpu_count(),
                             "fwd_tflops": round(4 * w.D * pair_flops * args.steps / t_f / 1e12, 6),
                             "bwd_tflops": round(10 * w.D * pair_flops * args.steps / t_b / 1e12,
                                                 6)},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="ltx_15300", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    rank, world, local = dist_setup(args.gpus)
    try:
        line = run_gpu(args, rank, world, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
