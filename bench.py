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
# NVIDIA's HGX B200 specification table gives FP16/BF16 tensor throughput as
# 36 PFLOPS for the 8-GPU board, a figure stated with 2:4 structured sparsity;
# per GPU and dense that is 36 / 8 / 2 = 2.25 PFLOPS.
DATASHEET_DENSE_BF16_TFLOPS = 2250.0
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
# workload: sizes, allowed pairs and algorithmic bytes
# ---------------------------------------------------------------------------
def seqlens(w: synth.Workload):
    """Per-sequence (seqlen_q, seqlen_k) lists of a workload."""
    if w.packed:
        return synth.varlen_seqlens(synth.VARLEN_SEQLEN_SEED)
    return [w.Sq] * w.B, [w.Sk] * w.B


def pair_count(sq: int, sk: int, wl: int, wr: int, bottom_right: bool) -> int:
    """Allowed (query, key) pairs of one sequence, counted in closed form: row i
    sees keys max(0, i - L) .. min(sk - 1, i + R) with (L, R) the window of the
    AOTriton 0.15b release notes ("Bottom-Right Aligned Sliding Windows":
    L = wl - d, R = wr + d under the bottom-right diagonal, d = sk - sq; the
    causal sentinels mean (inf, 0) and (inf, d) and are never shifted).  This
    is the benchmark's own count; the tests pin it to the oracle's mask."""
    import numpy as np
    if sq <= 0 or sk <= 0:
        return 0
    d = sk - sq
    if wl == synth.CAUSAL_TOP_LEFT:
        L, R = None, 0
    elif wl == synth.CAUSAL_BOTTOM_RIGHT:
        L, R = None, d
    else:
        L = None if wl == synth.WINDOW_INF else (wl - d if bottom_right else wl)
        R = None if wr == synth.WINDOW_INF else (wr + d if bottom_right else wr)
    i = np.arange(sq, dtype=np.int64)
    lo = np.zeros(sq, dtype=np.int64) if L is None else np.maximum(i - L, 0)
    hi = np.full(sq, sk - 1, dtype=np.int64) if R is None else np.minimum(i + R, sk - 1)
    return int(np.maximum(hi - lo + 1, 0).sum())


def workload_flops(w: synth.Workload):
    """(forward FLOP, backward FLOP, allowed pairs) of one step on one GPU."""
    sq, sk = seqlens(w)
    n = w.H * sum(pair_count(a, b, w.window_left, w.window_right, w.bottom_right)
                  for a, b in zip(sq, sk))
    return 4 * w.D * n, 10 * w.D * n, n


def workload_bytes(w: synth.Workload):
    """Algorithmic HBM bytes of one launch of each kernel (every tensor read or
    written once; 16-bit Q, K, V, O, dO, dQ, dK, dV, fp32 LSE, delta and dQ
    accumulator).  Per (query row, head): forward Q + O (4D) + LSE (4); main
    backward Q + dO (4D), LSE + delta (8), accumulator read + write (8D);
    preprocess + conversion 14D + 4.  Per (key row, head): forward K + V (4D);
    main backward K + V + dK + dV (8D)."""
    sq, sk = seqlens(w)
    rq, rk, D = w.H * sum(sq), w.H * sum(sk), w.D
    return {"attn_fwd_kernel": rq * (4 * D + 4) + rk * 4 * D,
            "attn_bwd_kernel": rq * (12 * D + 8) + rk * 8 * D,
            "bwd_other": rq * (14 * D + 4)}


def fwd_kernel_name(w: synth.Workload, bias: bool) -> str:
    """The forward kernel the library runs for this workload: the CTA-pair
    kernel for dense calls with head dims above 64 (the value head dim a
    multiple of 16) and no window, bias or dropout, the one-CTA kernel
    otherwise (the dispatch rule of the forward launch)."""
    dense = not w.packed and w.window_left == synth.WINDOW_INF and w.window_right == synth.WINDOW_INF
    pair = dense and 64 < w.D <= 128 and w.D % 16 == 0 and not bias
    return "attn_fwd_pair_kernel" if pair else "attn_fwd_kernel"


def describe(w: synth.Workload):
    sq, sk = seqlens(w)
    layout = ("packed 1THD with cumulative seqlens, LSE TH" if w.packed
              else f"BHSD dense, LSE {'TH' if w.lse_th else 'HT'}")
    per_tensor = w.H * sum(sq) * w.D * 2
    return {"workload": f"{w.name}: {w.describe}, fwd+bwd", "B": w.B, "H": w.H, "Sq": w.Sq,
            "Sk": w.Sk, "D": w.D, "dtype": w.dtype, "total_q": sum(sq), "total_k": sum(sk),
            "window": [w.window_left, w.window_right],
            "diagonal": "bottom-right" if w.bottom_right else "top-left", "layout": layout,
            "l2": "working set larger than L2 (Q, O, dO, dQ each "
                  f"{per_tensor / 1e6:.0f} MB, K, V, dK, dV each "
                  f"{w.H * sum(sk) * w.D * 2 / 1e6:.0f} MB; L2 is 126 MB)"}


def bias_bytes(w: synth.Workload, pairs: int):
    """Algorithmic HBM bytes the additive bias adds (16-bit elements): the
    forward reads B on the allowed pairs; the backward reads it there and
    writes dB = dS over every (query, key) pair of each sequence (0 on the
    masked ones)."""
    sq, sk = seqlens(w)
    every = w.H * sum(a * b for a, b in zip(sq, sk))
    return {"attn_fwd_kernel": 2 * pairs, "attn_bwd_kernel": 2 * pairs + 2 * every}


class Step:
    """Device buffers and the two C-ABI calls of one step."""

    def __init__(self, w: synth.Workload, dev, bias: bool = False):
        from scaled_dot_product_12_b200 import binding as B
        self.B = B
        self.w = w
        dtype = synth.DTYPES[w.dtype]
        if w.packed:
            sq, sk = seqlens(w)
            cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
            q, k, v, do = synth.qkv_do((int(cu_q[-1]), w.H, w.D), (int(cu_k[-1]), w.H, w.D),
                                       w.seed, dtype)
            self.host = {"q": q, "k": k, "v": v, "do": do, "cu_q": cu_q, "cu_k": cu_k}
            self.cu_q, self.cu_k = cu_q.to(dev), cu_k.to(dev)
            self.kw = dict(cu_seqlens_q=self.cu_q, cu_seqlens_k=self.cu_k, max_seqlen_q=max(sq),
                           max_seqlen_k=max(sk), lse_layout="TH")
        else:
            q, k, v, do = synth.qkv_do((w.B, w.H, w.Sq, w.D), (w.B, w.H, w.Sk, w.D), w.seed, dtype)
            self.host = {"q": q, "k": k, "v": v, "do": do}
            self.cu_q = self.cu_k = None
            self.kw = dict(lse_layout="TH" if w.lse_th else "HT")
        self.q, self.k, self.v, self.do = (t.to(dev) for t in (q, k, v, do))
        self.scale = w.D ** -0.5
        self.window = (w.window_left, w.window_right)
        self.o = torch.empty_like(self.q)
        pr = B.Problem(self.q, self.k, self.scale, self.window, w.bottom_right,
                       self.kw.get("cu_seqlens_q"), self.kw.get("cu_seqlens_k"),
                       self.kw.get("max_seqlen_q"), self.kw.get("max_seqlen_k"),
                       self.kw["lse_layout"])
        self.lse = torch.empty(pr.lse_shape(), dtype=torch.float32, device=dev)
        self.dq = torch.empty_like(self.q)
        self.dk = torch.empty_like(self.k)
        self.dv = torch.empty_like(self.v)
        self.bias = self.dbias = None
        if bias:
            # [B, H, Sq, Sk] (largest lengths for packed inputs), drawn on the
            # device: N(0, 1) from a seeded device generator; rows are padded
            # to a multiple of 8 elements (16-byte row strides)
            pitch = (pr.Sk + 7) // 8 * 8
            shape = (pr.B, w.H, pr.Sq, pitch)
            g = torch.Generator(device=dev).manual_seed(w.seed + 1)
            self.bias = torch.randn(shape, generator=g, device=dev,
                                    dtype=torch.float32).to(dtype)[..., :pr.Sk]
            self.dbias = torch.empty(shape, device=dev, dtype=dtype)[..., :pr.Sk]
            self.kw["bias"] = self.bias
        self.bp = B.bwd_params(self.do, self.q, self.k, self.v, self.o, self.lse, pr, self.dq,
                               self.dk, self.dv, bias=self.bias, dbias=self.dbias)
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
                  bottom_right=self.w.bottom_right, out=self.o, lse=self.lse, stream=stream,
                  **self.kw)
        if ev is not None:
            ev[1].record(stream)
            self.bp.main_kernel_events[0] = ev[2].cuda_event
            self.bp.main_kernel_events[1] = ev[3].cuda_event
        else:
            self.bp.main_kernel_events[0] = None
            self.bp.main_kernel_events[1] = None
        B._check("attn_bwd", B.lib().attn_bwd(ctypes.byref(self.bp), stream.cuda_stream))


def kernel_roofline(name, flops, nbytes, ms, peak_tflops, hbm_gbs):
    """Achieved rate of one kernel against the roofline that bounds it: the
    tensor pipe when flops / peak exceeds bytes / bandwidth, else HBM."""
    t_tensor = flops / (peak_tflops * 1e12)
    t_hbm = nbytes / (hbm_gbs * 1e9)
    if t_tensor >= t_hbm:
        ach = flops / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "kernel": name, "achieved": round(ach, 1), "peak": peak_tflops,
                "unit": "TFLOP/s", "frac": round(ach / peak_tflops, 4)}
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": name, "achieved": round(ach, 1), "peak": hbm_gbs,
            "unit": "GB/s", "frac": round(ach / hbm_gbs, 4)}


def run_gpu(args, rank, world, local):
    from scaled_dot_product_12_b200 import binding as B
    w = synth.ALL_WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    step = Step(w, dev, bias=args.bias)
    stream = torch.cuda.Stream(dev)
    fwd_flops, bwd_flops, pairs = workload_flops(w)
    nbytes = workload_bytes(w)
    if args.bias:
        for kname, extra in bias_bytes(w, pairs).items():
            nbytes[kname] += extra
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
    # GEMM figure while the SM clock stayed at its maximum, the sustained one
    # once the clock was lowered.  Both fractions are reported.
    burst = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    hbm = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    lowered = clock_lowered(clock_summary)
    peak = sustained if lowered else burst
    fwd_tf = fwd_flops / (fwd_ms * 1e-3) / 1e12
    bwd_tf = bwd_flops / (main_ms * 1e-3) / 1e12
    if main_ms >= fwd_ms:
        roof = kernel_roofline("attn_bwd_kernel", bwd_flops, nbytes["attn_bwd_kernel"], main_ms,
                               peak, hbm)
    else:
        roof = kernel_roofline(fwd_kernel_name(w, args.bias), fwd_flops, nbytes["attn_fwd_kernel"],
                               fwd_ms, peak, hbm)
    roof["peak_source"] = peak_source(peak_src, lowered, clock_summary)
    roof["traffic"] = load_traffic(roof["kernel"], w.name)

    # ---- end to end through the C ABI with host buffers ----
    if args.bias:
        e2e = {"skipped": "bias runs measure the kernels only (the bias and its gradient "
                          "would add two Sq x Sk tensors per head to every copy)"}
    else:
        e2e = run_e2e(step, stream, dev, min(args.steps, 5), flops, world)

    def per_kernel(tf, ms, nb):
        return {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_of_peak": round(tf / peak, 4),
                "frac_of_burst": round(tf / burst, 4), "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                "frac_of_hbm": round(nb / (ms * 1e-3) / 1e9 / hbm, 4)}

    line = {
        "metric": "attention TFLOP/s (fwd+bwd, unmasked FLOPs)", "value": round(value, 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp16",
        "data": "synthetic: i.i.d. N(0,1) Q, K, V, dO from a fixed seed",
        "config": dict(describe(w), **({"bias": "additive bias [B, H, Sq, Sk] N(0, 1) in the "
                                                "input dtype, and its gradient"}
                                       if args.bias else {})),
        "fwd": per_kernel(fwd_tf, fwd_ms, nbytes["attn_fwd_kernel"]),
        "bwd_main": per_kernel(bwd_tf, main_ms, nbytes["attn_bwd_kernel"]),
        "bwd_other_ms": round(ms_step - fwd_ms - main_ms, 4),
        # The delta preprocess and the dQ conversion are HBM-bound: their
        # algorithmic bytes over the rest of the step (both kernels and the
        # gaps between launches) give a lower bound on their bandwidth.
        "bwd_other": other_bandwidth(nbytes["bwd_other"] * world, ms_step - fwd_ms - main_ms, hbm),
        "frac_of_peak": {"measured_burst": round(value / world / burst, 4),
                         "measured_sustained": round(value / world / sustained, 4),
                         "datasheet_dense": round(value / world / DATASHEET_DENSE_BF16_TFLOPS, 4)},
        "roofline": roof,
        "gpu_launches": 4 * args.steps,
        "clocks": clock_summary,
        "e2e": e2e,
        "allowed_pairs": pairs,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.bias:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def other_bandwidth(nbytes, ms, hbm_gbs):
    """Preprocess reads O, dO (2 x 2D bytes per row and head) and writes delta
    (4) and the zeroed fp32 dQ accumulator (4D); the conversion reads the
    accumulator (4D) and writes dQ (2D): (14 D + 4) bytes per row and head."""
    gbs = nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None
    return {"ms": round(ms, 4), "bytes": nbytes, "gbs": round(gbs, 1) if gbs else None,
            "peak_gbs": hbm_gbs, "frac": round(gbs / hbm_gbs, 4) if gbs else None}


def clock_lowered(clocks):
    """True if the SM clock was lowered during the timed region, whatever the
    cause: a median SM clock more than 3 % under the maximum.  A throttle flag
    alone, with the clock still at its maximum, leaves the burst figure the
    right denominator."""
    mhz, top = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    return bool(mhz and top and mhz < 0.97 * top)


def peak_source(src, lowered, clocks):
    if not lowered:
        return (f"{src} bf16_tflops (burst: the SM clock stayed at its maximum during the "
                "timed region)")
    seen = [r for r in clocks.get("reasons", []) if r not in ("gpu_idle",)]
    return (f"{src} bf16_tflops_sustained (median SM clock {clocks.get('sm_mhz')} MHz against "
            f"a {clocks.get('sm_max_mhz')} MHz maximum; throttle reasons seen: "
            f"{', '.join(seen) if seen else 'none'})")


# The sources each kernel is compiled from (its .cu file and the headers it
# includes): committed counters of a kernel stay valid while these are unchanged.
_BWD_SOURCES = ("common.cuh", "mask.cuh", "fwd.h", "bwd.cu")
KERNEL_SOURCES_BY_KERNEL = {
    "attn_fwd_kernel": ("common.cuh", "mask.cuh", "fwd.h", "fwd.cu"),
    "attn_fwd_pair_kernel": ("common.cuh", "fwd.h", "fwd_pair.cu"),
    "attn_bwd_kernel": _BWD_SOURCES,
    "attn_bwd_pre_kernel": _BWD_SOURCES,
    "attn_dq_convert_kernel": _BWD_SOURCES,
}
KERNEL_SOURCES = tuple(sorted({f for v in KERNEL_SOURCES_BY_KERNEL.values() for f in v}))


def _code_only(text: str) -> str:
    """C / C++ source without comments and with runs of whitespace collapsed:
    what the compiler sees, so an edit of a comment keeps the hash."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":  # string or character literal, copied whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernels_sha256(kernel=None):
    """Hash of a kernel's sources (comments and layout ignored; all kernel
    sources when `kernel` is None), to tie committed counters to a build."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES_BY_KERNEL[kernel] if kernel else KERNEL_SOURCES:
        with open(os.path.join(ROOT, "scaled_dot_product_12_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
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
    if kernel not in KERNEL_SOURCES_BY_KERNEL:
        return None
    if d.get("kernels_sha256", {}).get(kernel) != kernels_sha256(kernel):
        return None
    return d.get("bytes_per_launch", {}).get(f"{kernel}:{workload}")


def e2e_groups(w: synth.Workload, n_groups: int):
    """Slices along which the end-to-end step is pipelined: batches when there
    are several (LSE rows of a batch are contiguous in HT layout), else heads
    of the single batch.  Packed workloads, and steps whose inputs are under
    64 MB (latency-bound: more calls would only add host time), run as one
    group."""
    in_bytes = 2 * w.D * w.H * w.B * (2 * w.Sq + 2 * w.Sk)
    if w.packed or n_groups <= 1 or in_bytes < (64 << 20):
        return None, [slice(None)]
    dim, size = (0, w.B) if w.B > 1 else (1, w.H)
    n = min(n_groups, size)
    edges = [size * g // n for g in range(n + 1)]
    return dim, [slice(edges[g], edges[g + 1]) for g in range(n) if edges[g + 1] > edges[g]]


def run_e2e(step: Step, stream, dev, n, flops, world, n_groups: int = 4):
    """The same work through the same C-ABI calls from pinned HOST buffers:
    every step copies Q, K, V, dO (and the cumulative seqlens of packed inputs)
    in and O, LSE, dQ, dK, dV out inside the timed region.  Dense workloads
    are cut into groups of batches (or of heads when B = 1), each a forward and
    backward call of its own, and pipelined over three streams: group g's
    inputs copy in while group g - 1 computes and group g - 2's outputs copy
    out."""
    w = step.w
    B = step.B
    host_in = {k: v.pin_memory() for k, v in step.host.items()}
    outs = ["o", "lse", "dq", "dk", "dv"]
    host_out = {k: torch.empty(getattr(step, k).shape, dtype=getattr(step, k).dtype,
                               pin_memory=True) for k in outs}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    dim, groups = e2e_groups(w, n_groups)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def part(t, g):
        if dim is None:
            return t
        return t[g] if dim == 0 else t[:, g]

    kw = dict(sm_scale=step.scale, window=step.window, bottom_right=w.bottom_right, **step.kw)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    done_in = [ev() for _ in groups]
    done_fb = [ev() for _ in groups]
    done_out = [ev() for _ in groups]
    started = [False] * len(groups)

    def one_step():
        for gi, g in enumerate(groups):
            with torch.cuda.stream(s_in):
                if started[gi]:
                    s_in.wait_event(done_fb[gi])  # last step's compute no longer reads them
                for name, t in host_in.items():
                    dst = getattr(step, name)
                    if name in ("cu_q", "cu_k"):
                        dst.copy_(t, non_blocking=True)
                    else:
                        part(dst, g).copy_(part(t, g), non_blocking=True)
                done_in[gi].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(done_in[gi])
                if started[gi]:
                    stream.wait_event(done_out[gi])  # last step's outputs have left
                o, lse = part(step.o, g), part(step.lse, g)
                q, k, v, do = (part(getattr(step, x), g) for x in ("q", "k", "v", "do"))
                B.forward(q, k, v, out=o, lse=lse, stream=stream, **kw)
                B.backward(do, q, k, v, o, lse, dq=part(step.dq, g), dk=part(step.dk, g),
                           dv=part(step.dv, g), workspace=step.ws, stream=stream, **kw)
                done_fb[gi].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_fb[gi])
                for name in outs:
                    part(host_out[name], g).copy_(part(getattr(step, name), g), non_blocking=True)
                done_out[gi].record(s_out)
            started[gi] = True

    one_step()  # warm-up: the same work, untimed
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    t0.record(s_in)
    for _ in range(n):
        one_step()
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1) / n, world)
    total = sum_over_ranks(flops, world)
    return {"value": round(total / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipeline": (f"{len(groups)} groups of {'batches' if dim == 0 else 'heads'} over "
                         "copy-in, compute and copy-out streams") if dim is not None
            else "one group (copy in, compute, copy out in order)"}


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
    """Inputs of a bounded sample and its FLOP count (14*D per allowed pair,
    counted with the oracle's own mask): head 0 of the first (batch or packed)
    sequence, its first `rows` query rows (all rows if rows <= 0) against all
    of its keys.  A prefix of the query rows is itself a problem with the same
    mask rows only when the window does not depend on seqlen_q (top-left
    windows, no mask); otherwise the whole sequence is the sample."""
    import numpy as np

    from oracle import attn_ref as ref
    dtype = synth.DTYPES[w.dtype]
    sq, sk = seqlens(w)
    if w.packed:
        q, k, v, do = synth.qkv_do((sum(sq), w.H, w.D), (sum(sk), w.H, w.D), w.seed, dtype)
        f = lambda t, n: t[:n, 0].float().numpy().astype(np.float64)  # noqa: E731
        qn, kn, vn, don = f(q, sq[0]), f(k, sk[0]), f(v, sk[0]), f(do, sq[0])
    else:
        q, k, v, do = synth.qkv_do((w.B, w.H, w.Sq, w.D), (w.B, w.H, w.Sk, w.D), w.seed, dtype)
        f = lambda t: t[0, 0].float().numpy().astype(np.float64)  # noqa: E731
        qn, kn, vn, don = f(q), f(k), f(v), f(do)
    no_mask = w.window_left == synth.WINDOW_INF and w.window_right == synth.WINDOW_INF
    depends_on_sq = w.window_left == synth.CAUSAL_BOTTOM_RIGHT or (
        w.bottom_right and w.window_left != synth.CAUSAL_TOP_LEFT and not no_mask)
    n = qn.shape[0] if rows <= 0 or depends_on_sq else min(rows, qn.shape[0])
    qn, don = qn[:n], don[:n]
    pairs = ref.allowed_count(n, kn.shape[0], w.window_left, w.window_right, w.bottom_right)
    return (qn, kn, vn, don), 14 * w.D * pairs


def oracle_step(w, inputs):
    """One oracle forward and backward of the sample; returns their wall
    times (s)."""
    from oracle import attn_ref as ref
    qn, kn, vn, don = inputs
    args = (w.D ** -0.5, w.window_left, w.window_right, w.bottom_right)
    t0 = time.perf_counter()
    ref.forward(qn, kn, vn, *args)
    t1 = time.perf_counter()
    ref.backward(qn, kn, vn, don, *args)
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
            "sample": f"fp64 NumPy oracle, forward + backward of head 0 of the first sequence "
                      f"({inputs[0].shape[0]} query rows x {inputs[1].shape[0]} keys, "
                      f"{flops / 1e9:.1f} GFLOP at 14*D per allowed pair), {dt:.1f} s on "
                      f"{os.cpu_count()} host cores"}


def run_reference(args, rank, world):
    """--impl reference: the oracle as it stands, timed on the host cores."""
    w = synth.ALL_WORKLOADS[args.workload]
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
    sample = (f"each step: fp64 NumPy oracle forward + backward of head 0 of the first sequence, "
              f"its first {inputs[0].shape[0]} query rows against all {inputs[1].shape[0]} keys "
              f"({flops / 1e9:.2f} GFLOP)")
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
    ap.add_argument("--workload", default="ltx_15300", choices=sorted(synth.ALL_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bias", action="store_true",
                    help="add an additive bias [B, H, Sq, Sk] to the step and write its gradient "
                         "(kernels only: no end-to-end or CPU leg)")
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
