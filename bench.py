"""Benchmark of the SVDQuant W4A4 linear layer on B200.

One step = one pass of the per-call path over one batch of tokens:
svdq_quantize_act (smoothing + NVFP4 quantization + fused low-rank
down-projection) then svdq_linear (tcgen05 FP4 GEMM + fused up-projection),
with X already resident in device memory. Metric: effective TFLOPS,
FLOPs = 2MNK + 2Mr(K+N) per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores

Multi-GPU (launched by torchrun, one rank per GPU): every rank runs the layer
on its own batch of tokens with the same weights (token rows are independent:
no data-path collective); the step time is the max over ranks, the value the
FLOPs of all ranks over that time (weak scaling).

Timing: W untimed warm-up steps, then K steps timed with CUDA events on the
launching stream around the whole block (the library launches each kernel so
that its prologue overlaps the end of the previous one, as in a network of
layers); the same K steps are then timed again with events around each kernel
for the per-kernel rooflines and the step percentiles (events between kernels
serialize them). Steps rotate over copies of X and of the prepared weights
whose total exceeds twice the 126 MB L2, so every step reads its inputs from
HBM (as a network whose layers each have their own weights would).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a4_diffusion_model_b200 import synth  # noqa: E402

METRIC = "SVDQuant W4A4 linear effective TFLOPS (2MNK + 2Mr(K+N)) per layer call, FLUX shapes"
DEFAULT_WORKLOAD = synth.FLUX_QKV.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_PER_BF16 = 4.0        # nominal dense FP4 : BF16 tensor throughput ratio on B200 (9 : 2.25 PFLOP/s)
DATASHEET_FP4_TFLOPS = 9000.0


def parse():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    p.add_argument("--codec", default="nvfp4", choices=["nvfp4", "int4"],
                   help="int4: the INT4 W4A4 variant (64-element groups, fp16 scales) of the same layer")
    p.add_argument("--no-extras", action="store_true", help="skip the cuBLAS / unfused / rank-0 / e2e / CPU legs")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    p.add_argument("--extra-json", default=None, help="append per-leg details to this JSONL file")
    p.add_argument("--deltaquant-only", action="store_true",
                   help="time only the DeltaQuant encoder on the bench's video latent (one JSON line; for profiling)")
    return p.parse_args()


# --------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


L2_BYTES = 126 * 1024 * 1024


def weight_bytes(P) -> int:
    return sum(t.numel() * t.element_size() for t in (P.Qr, P.Sr, P.L1p, P.L2t, P.lam, P.inv_lam) if t is not None)


def clone_weights(P):
    """A copy of prepared weights in fresh device buffers."""
    return dataclasses.replace(P, **{f: (getattr(P, f).clone() if getattr(P, f) is not None else None)
                                     for f in ("Qr", "Sr", "L1p", "L2t", "lam", "inv_lam")})


def quantize_bytes(w: synth.Workload) -> int:
    """Algorithmic HBM bytes of one quantize launch: read X, inv_lambda, L1p;
    write codes, scales (rows padded to 128) and T."""
    Mp = (w.M + 127) // 128 * 128
    return 2 * w.M * w.K + 4 * w.K + 2 * w.rank * w.K + w.M * w.K // 2 + Mp * w.K // 16 + 2 * w.M * w.rank


def gemm_flops(w: synth.Workload) -> int:
    """Algorithmic FLOPs of one GEMM launch: 2MNK (FP4) + 2MrN (fused up-projection)."""
    return 2 * w.M * w.N * w.K + 2 * w.M * w.rank * w.N


GEMM_SOURCES = ("svdq_gemm.cuh", "svdq_gemm_pair.cuh", "svdq_gemm_common.cuh", "svdq_gemm_qnext.cuh", "svdq_ptx.cuh",
                "svdq_quant.cuh", "svdq_quant_tma.cuh")
QUANT_SOURCES = ("svdq_quant_tma.cuh", "svdq_quant.cuh", "svdq_ptx.cuh")
INT4_SOURCES = ("svdq_int4.cuh", "svdq_gemm_common.cuh", "svdq_ptx.cuh")


def quantize_bytes_int4(w: synth.Workload) -> int:
    """Algorithmic HBM bytes of one INT4 quantize launch: read X, inv_lambda,
    L1p; write one code byte per element, fp32 scales (rows padded to 128), T."""
    Mp = (w.M + 127) // 128 * 128
    return 2 * w.M * w.K + 4 * w.K + 2 * w.rank * w.K + w.M * w.K + Mp * (w.K // 64) * 4 + 2 * w.M * w.rank


def kernel_source_hash(sources=GEMM_SOURCES) -> str:
    """Hash of a kernel's sources: ties a committed ncu traffic figure to the
    kernel version it was measured on."""
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "w4a4_diffusion_model_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def gemm_kernel_name(w: synth.Workload) -> str:
    return "svdq_gemm_pair_kernel" if w.N % 256 == 0 else "svdq_gemm_kernel"


def profiled_traffic(summary: str, sources):
    """DRAM bytes per launch from a committed ncu summary under profiles/, if
    it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    src_hash = kernel_source_hash(sources)
    with open(p) as f:
        for line in f:
            if line.startswith("traffic_bytes_per_launch:"):
                parts = line.split()
                if len(parts) >= 3 and parts[2] == src_hash:
                    return float(parts[1])
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while active.
    summary(t0, t1) keeps the samples taken inside the host-time window
    [t0, t1] (the timed region); if that window is shorter than the sampling
    period it falls back to every sample taken while the GPU was loaded."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def n_samples(self) -> int:
        try:
            with open(self.path) as f:
                return sum(1 for _ in f)
        except Exception:
            return 0

    def summary(self, t0: float, t1: float, t_load: float):
        if self.proc is None or not self.path:
            return None
        import datetime
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if len(inside) < 2:
            inside = [r for r in rows if t_load <= r[0] <= t1]
            window = "spin-up + timed region (timed region shorter than the 200 ms sampling period)"
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, _, flags in inside for i, fl in enumerate(flags) if fl == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "window": window}


def smi_index(local: int) -> str:
    """nvidia-smi --id of the GPU behind CUDA device `local`."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


# --------------------------------------------------------------------------- CPU oracle leg
def oracle_sample(w: synth.Workload, X_cpu: torch.Tensor, W_cpu: torch.Tensor, rows=64, cols=512, codec="nvfp4"):
    """Set up the oracle's per-call path on a bounded sample: `rows` token rows
    and `cols` output channels of the layer, full K. Returns (fn, flops)."""
    import oracle as O  # only the CPU-baseline / reference legs use the oracle

    rng = np.random.default_rng(w.seed + 17)
    r_idx = np.sort(rng.choice(w.M, min(rows, w.M), replace=False))
    c_idx = np.sort(rng.choice(w.N, min(cols, w.N), replace=False))
    Xn = X_cpu.float().numpy().astype(np.float64)
    Wn = W_cpu.float().numpy().astype(np.float64)
    amax = O.channel_amax(Xn)
    lam32, inv32 = O.smoothing_lambda(amax, Wn, w.alpha)
    What_c = lam32.astype(np.float64)[:, None] * Wn[c_idx].T
    U, S, Vt = np.linalg.svd(What_c, full_matrices=False)
    L1p = O.bf16(U[:, :w.rank] * S[:w.rank] / lam32.astype(np.float64)[:, None])
    L2 = O.bf16(Vt[:w.rank])
    R32, qr, sr = O.residual_quantize(Wn[c_idx], lam32, L1p, L2)
    Xs = Xn[r_idx]

    def fn():
        qx, sx, T = O.quantize_act(Xs, inv32, L1p)
        return O.linear(qx, sx, T, qr, sr, L2)

    if codec == "int4":
        qr4, sr4 = O.quantize_int4(R32.T)
        deq_r = O.dequantize_int4(qr4, sr4)

        def fn():  # noqa: F811
            xhat = Xs.astype(np.float32) * inv32.astype(np.float32)[None, :]
            qx4, sx4 = O.quantize_int4(xhat)
            return O.dequantize_int4(qx4, sx4) @ deq_r.T + (Xs @ L1p) @ L2

    m, n = len(r_idx), len(c_idx)
    flops = 2 * m * n * w.K + 2 * m * w.rank * (w.K + n)
    sample = (f"oracle per-call path ({codec} quantize + down-projection + dequantized fp64 GEMM + up-projection) "
              f"on {m} token rows x {n} output channels x K={w.K} of {w.name}; prepare excluded")
    return fn, flops, sample


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def square_gemm_rate(S, dev, n=8192, reps=10) -> dict:
    """The GEMM alone at rank 0 on a large square shape (n x n x n): the best
    FP4 rate this kernel reaches -- an achieved figure, not a peak."""
    g = torch.Generator(device="cpu").manual_seed(7)
    X = (torch.randn(n, n, generator=g) / 4).to(torch.bfloat16).to(dev)
    W = (torch.randn(n, n, generator=g) / n ** 0.5).to(torch.bfloat16).to(dev)
    P = S.svdq_prepare_weights(W, S.svdq_channel_amax(X), 0.5, 0)
    Qx, Sx, _ = S.svdq_quantize_act(X, P.inv_lam, None, 0, n)
    Y = torch.empty(n, n, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        S.svdq_linear(Qx, Sx, None, P, out=Y)
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        S.svdq_linear(Qx, Sx, None, P, out=Y)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    S.svdq_check()
    return {"shape": f"{n}x{n}x{n}", "ms": round(best, 4), "tflops": round(2 * n ** 3 / (best * 1e-3) / 1e12, 1),
            "note": "achieved, not peak"}


def time_cpu(fn, flops, seconds):
    fn()  # warm
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return flops * n / el / 1e12, n, el


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    X, W = synth.generate(w)
    fn, flops, sample = oracle_sample(w, X, W, codec=args.codec)
    for _ in range(args.warmup):
        fn()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = flops * len(times) / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot / len(times), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "rank": w.rank, "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU leg
def int4_extras(args, w, step4, X, Y, X_cpu, W_cpu, flops_step, world, rank_id, timed):
    """e2e and CPU baseline of the INT4 variant: each step uploads its X from
    pinned host memory into the first input set's buffer, runs the layer and
    downloads Y (one step at a time)."""
    n_x = max(5, args.steps // 2)
    stream = torch.cuda.current_stream()
    X_host = X_cpu.pin_memory()
    Y_host = torch.empty(w.M, w.N, dtype=torch.bfloat16).pin_memory()

    def e2e_step(i, ev):
        ev[0].record(stream)
        X.copy_(X_host, non_blocking=True)
        step4(0)
        Y_host.copy_(Y, non_blocking=True)
        ev[1].record(stream)
        ev[2].record(stream)
    ke, _ = timed(n_x, e2e_step)
    e2e_ms = aggregate_max(sum(ke), world) / n_x
    e2e = {"value": round(flops_step * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2,
           "ms_per_step": round(e2e_ms, 4), "pipeline": "one step at a time"}
    cpu = None
    if rank_id == 0 and world == 1:
        fn, fl, sample = oracle_sample(w, X_cpu, W_cpu, codec="int4")
        v, n, el = time_cpu(fn, fl, args.cpu_seconds)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample, "repeats": n, "seconds": round(el, 2)}
    return e2e, cpu


def flux_shape_summary(S, w: synth.Workload, dev, n: int, fp4_peak: float) -> dict:
    """Layer and GEMM figures of another FLUX projection, timed like the main
    workload: rotating input sets larger than twice the L2, the layer block with
    one event pair (dependent launches overlap), the GEMM per launch (events
    around each kernel) and back to back. Weights are prepared by the library."""
    X_cpu, W_cpu = synth.generate(w)
    X, W = X_cpu.to(dev), W_cpu.to(dev)
    P = S.svdq_prepare_weights(W, S.svdq_channel_amax(X), w.alpha, w.rank)
    del W
    set_bytes = X.numel() * 2 + weight_bytes(P)
    n_sets = max(2, min(16, -(-2 * L2_BYTES // set_bytes)))
    sets = [(X, P)] + [(X.clone(), clone_weights(P)) for _ in range(n_sets - 1)]
    Qx = torch.empty(w.M, w.K // 2, dtype=torch.uint8, device=dev)
    Sx = torch.empty(S.svdq_act_sizes(S.LayerShape(w.M, w.K, w.N, w.rank))[1], dtype=torch.uint8, device=dev)
    T = torch.empty(w.M, w.rank, dtype=torch.bfloat16, device=dev)
    Y = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def quant(i):
        X_, P_ = sets[i % n_sets]
        S.svdq_quantize_act(X_, P_.inv_lam, P_.L1p, w.rank, w.N, S.SVDQ_FUSED, out=(Qx, Sx, T))

    def gemm(i):
        S.svdq_linear(Qx, Sx, T, sets[i % n_sets][1], S.SVDQ_FUSED, out=Y)

    def block(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    for i in range(5):
        quant(i)
        gemm(i)
    layer_ms = block(lambda i: (quant(i), gemm(i)))
    gemm_block = block(gemm)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    torch.cuda.synchronize()
    torch.cuda._sleep(2_000_000)
    for i in range(n):
        ev[i][0].record(stream)
        quant(i)
        ev[i][1].record(stream)
        gemm(i)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    S.svdq_check()
    q_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    g_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    g_tf = gemm_flops(w) / (g_ms * 1e-3) / 1e12
    gb_tf = gemm_flops(w) / (gemm_block * 1e-3) / 1e12
    return {"workload": w.name, "layer_ms": round(layer_ms, 4),
            "layer_tflops": round(w.flops() / (layer_ms * 1e-3) / 1e12, 1),
            "quantize_ms": round(q_ms, 4), "quantize_gbs": round(quantize_bytes(w) / (q_ms * 1e-3) / 1e9, 1),
            "gemm_ms": round(g_ms, 4), "gemm_tflops": round(g_tf, 1),
            "gemm_frac": round(g_tf / fp4_peak, 4), "gemm_frac_datasheet_9pf": round(g_tf / DATASHEET_FP4_TFLOPS, 4),
            "gemm_block_ms": round(gemm_block, 4), "gemm_block_tflops": round(gb_tf, 1),
            "gemm_block_frac": round(gb_tf / fp4_peak, 4),
            "gemm_block_frac_datasheet_9pf": round(gb_tf / DATASHEET_FP4_TFLOPS, 4),
            "fp4_peak_tflops": round(fp4_peak, 1), "input_sets": n_sets}


def scale_group_stats(S, native, rows: int, K: int) -> dict:
    """Counts over the E4M3 group scales of a native scale buffer (rows x K/16
    groups): zero (an all-zero group, or amax / 6 below half the smallest
    subnormal: every code +0), subnormal (exponent field 0: fewer significant
    bits in the scale) and saturated (448, the largest finite E4M3 value: the
    group's amax / 6 reached it and its largest values may clip)."""
    c = S.svdq_scales_to_canonical(native, rows, K)
    zero = int((c == 0).sum())
    return {"groups": int(c.numel()), "zero": zero, "subnormal": int(((c & 0x78) == 0).sum()) - zero,
            "saturated": int((c == 0x7E).sum())}


def deltaquant_bytes(F: int, H: int, W: int, C: int) -> int:
    """Algorithmic HBM bytes of one DeltaQuant encode: read the bf16 tokens;
    write the E4M3 cores, the packed delta codes and their native scales."""
    T = F * H * W
    blocks = ((F + 1) // 2) * ((H + 1) // 2) * ((W + 1) // 2)
    return 2 * T * C + blocks * C + T * C // 2 + (T + 127) // 128 * (C // 64) * 512


def deltaquant_summary(S, dev, n: int, dims=(16, 32, 48), C: int = 3072) -> dict:
    """The DeltaQuant encoder on a video latent (smooth synthetic tokens),
    launched back to back over two copies of the input (more than twice the
    L2) with one event pair around the block."""
    F, H, W = dims
    X0 = synth.smooth_video(F, H, W, C, seed=77).to(dev)
    Xs = [X0, X0.clone()]
    cb, _, sb = S.svdq_deltaquant_sizes(F, H, W, C)
    out = (torch.empty(cb // C, C, dtype=torch.uint8, device=dev),
           torch.empty(F * H * W, C // 2, dtype=torch.uint8, device=dev),
           torch.empty(sb, dtype=torch.uint8, device=dev))
    for i in range(3):
        S.svdq_deltaquant_encode(Xs[i % 2], dims, out=out)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    torch.cuda._sleep(2_000_000)
    e0.record(stream)
    for i in range(n):
        S.svdq_deltaquant_encode(Xs[i % 2], dims, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    S.svdq_check()
    ms = e0.elapsed_time(e1) / n
    nbytes = deltaquant_bytes(F, H, W, C)
    return {"kernel": "deltaquant_encode_kernel", "video": f"{F}x{H}x{W} tokens x {C} channels, 2x2x2 blocks",
            "ms": round(ms, 4), "algorithmic_bytes": nbytes, "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}


def aggregate_max(value: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args):
    from w4a4_diffusion_model_b200 import svdq as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank_id = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    S.load()

    w = synth.WORKLOADS[args.workload]
    X_cpu, W_cpu = synth.generate(w)
    if rank_id > 0:          # each rank its own tokens, same weights
        X_cpu, _ = synth.generate(w.with_(seed=w.seed + 7919 * rank_id))
    X = X_cpu.to(dev)
    W = W_cpu.to(dev)

    # offline (untimed for the metric): calibration amax, smoothing, device SVD
    # split and residual encoding, all through the library
    amax = S.svdq_channel_amax(X)
    P0 = S.svdq_prepare_weights(W, amax, w.alpha, 0)
    torch.cuda.synchronize()
    e_prep = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    e_prep[0].record()
    P = S.svdq_prepare_weights(W, amax, w.alpha, w.rank)
    e_prep[1].record()
    torch.cuda.synchronize()
    prepare_ms = e_prep[0].elapsed_time(e_prep[1])

    int4 = args.codec == "int4"
    qx_b, sx_b, t_b = S.svdq_act_sizes(S.LayerShape(w.M, w.K, w.N, w.rank))

    def int4_act_buffers():
        """INT4 activation codes (one byte each) and group-major fp32 scales."""
        return (torch.empty(w.M, w.K, dtype=torch.uint8, device=dev),
                torch.empty(w.K // 64, (w.M + 127) // 128 * 128, dtype=torch.float32, device=dev))
    if int4:
        Qx, Sx = int4_act_buffers()
    else:
        Qx = torch.empty(w.M, w.K // 2, dtype=torch.uint8, device=dev)
        Sx = torch.empty(sx_b, dtype=torch.uint8, device=dev)
    T = torch.empty(w.M, w.rank, dtype=torch.bfloat16, device=dev) if w.rank else None
    Y = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    # L2: every step reads its own copy of X and of the prepared weights; the
    # copies together exceed twice the L2, so each step starts from HBM.
    set_bytes = X.numel() * 2 + weight_bytes(P)
    n_sets = max(2, min(16, -(-2 * L2_BYTES // set_bytes)))
    sets = [(X, P, P0)] + [(X.clone(), clone_weights(P), clone_weights(P0)) for _ in range(n_sets - 1)]
    l2_note = f"rotating {n_sets} input sets (X + prepared weights, {set_bytes / 1e6:.1f} MB each) > 2x L2"

    def make_step4(Qx_, Sx_):
        """One INT4 layer step on input set i (INT4 residual codes of every set,
        same smoothing and low-rank factors); events as in step()."""
        sets4 = [S.svdq_int4_prepare_weights(W, P_) for _, P_, _ in sets]

        def step4(i=0, ev=None):
            X_, P_, _ = sets[i % n_sets]
            if ev is not None:
                ev[0].record(stream)
            S.svdq_int4_quantize_act(X_, P_.inv_lam, P_.L1p, w.rank, w.N, out=(Qx_, Sx_, T))
            if ev is not None:
                ev[1].record(stream)
            S.svdq_int4_linear(Qx_, Sx_, T, sets4[i % n_sets], out=Y)
            if ev is not None:
                ev[2].record(stream)
        return step4, sets4
    step4 = make_step4(Qx, Sx)[0] if int4 else None

    def step(i=0, rank0=False, variant=S.SVDQ_FUSED, ev=None):
        if int4:
            return step4(i, ev)
        X_, P_, P0_ = sets[i % n_sets]
        if rank0:
            P_ = P0_
        r = P_.shape.rank
        if ev is not None:
            ev[0].record(stream)
        S.svdq_quantize_act(X_, P_.inv_lam, P_.L1p, r, w.N, variant, out=(Qx, Sx, T if r else None))
        if ev is not None:
            ev[1].record(stream)
        S.svdq_linear(Qx, Sx, T if r else None, P_, variant, out=Y)
        if ev is not None:
            ev[2].record(stream)

    def timed_block(n, fn):
        """Device time of n consecutive steps with CUDA events only around the
        whole block, so consecutive kernels overlap as they do in a network of
        layers (each kernel's prologue runs while the previous kernel ends)."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def timed(n, fn, warm=3, nlegs=0):
        """Per-step CUDA events around the two kernels (for each of `nlegs`
        interleaved legs when nlegs > 0). A GPU-side delay first lets the host
        queue the steps ahead of the device."""
        def events():
            mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            return [mk() for _ in range(nlegs)] if nlegs else mk()
        for i in range(warm):      # untimed: first-call setup (library handles, heuristics) stays out
            fn(i, events())
        evs = [events() for _ in range(n)]
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        for i in range(n):
            fn(i, evs[i])
        torch.cuda.synchronize()

        def split(ev_list):
            return ([e[0].elapsed_time(e[1]) for e in ev_list], [e[1].elapsed_time(e[2]) for e in ev_list])
        if nlegs:
            return [split([evs[i][leg] for i in range(n)]) for leg in range(nlegs)]
        return split(evs)

    with ClockSampler(smi_index(local)) as clk:
        # spin-up: keep the GPU loaded until the sampler reports, then warm up
        t_load = time.time()
        t_end = t_load + 1.5
        while time.time() < t_end and (clk.n_samples() < 2 or time.time() < t_load + 0.6):
            for i in range(20):
                step(i)
            torch.cuda.synchronize()
        for i in range(args.warmup):
            step(i)
        S.svdq_check()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        block_ms = timed_block(args.steps, lambda i: step(i))
        # the same steps with events between the two kernels, for the per-kernel
        # times of the two rooflines (the events serialize the kernels)
        k1, k2 = timed(args.steps, lambda i, ev: step(i, ev=ev), warm=0)
        torch.cuda.synchronize()
        t1 = time.time()
        if world > 1:
            torch.distributed.barrier()
        time.sleep(0.25)
    S.svdq_check()
    clocks = clk.summary(t0 - 0.2, t1 + 0.2, t_load)

    step_ms = [a + b for a, b in zip(k1, k2)]
    total_ms = aggregate_max(block_ms, world)
    ms_per_step = total_ms / args.steps
    flops_step = w.flops()
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    # the GEMM is timed alone inside a region of a few ms, so the burst bf16
    # figure is the matching denominator; the sustained one and the 9 PFLOP/s
    # datasheet figure are reported beside it
    fp4_peak = FP4_PER_BF16 * peaks["bf16_tflops"]
    fp4_sustained = FP4_PER_BF16 * peaks["bf16_tflops_sustained"]
    k2_ms = statistics.mean(k2)
    k1_ms = statistics.mean(k1)
    achieved = gemm_flops(w) / (k2_ms * 1e-3) / 1e12
    traffic = profiled_traffic(f"svdq_gemm_{w.name}.md", GEMM_SOURCES)
    sm_hz = ((clocks or {}).get("sm_mhz") or 1900) * 1e6
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    # INT4 GEMM bound: the rescale's two fp32 operations per output element and
    # 64-group (128 GEMM flops each), 128 fp32 lanes per SM at the sampled clock
    alu_peak = 64 * 128 * n_sm * sm_hz / 1e12
    fp8_peak = 2 * peaks["bf16_tflops_sustained"]
    roofline = {"bound": "tensor", "kernel": gemm_kernel_name(w), "achieved": round(achieved, 2),
                "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp4_peak, 4),
                "traffic": traffic,
                "frac_datasheet_9pf": round(achieved / DATASHEET_FP4_TFLOPS, 4),
                "frac_4x_sustained_bf16": round(achieved / fp4_sustained, 4),
                "peak_note": f"dense FP4 = {FP4_PER_BF16:g} x {peak_src} burst bf16 "
                             f"{peaks['bf16_tflops']:.1f} TFLOP/s (the kernel is timed alone, per launch); "
                             f"vs {DATASHEET_FP4_TFLOPS:g} TFLOP/s datasheet: {achieved / DATASHEET_FP4_TFLOPS:.4f}; "
                             f"vs {FP4_PER_BF16:g} x sustained bf16: {achieved / fp4_sustained:.4f}"}
    if int4:
        roofline = {"bound": "alu", "kernel": "svdq_int4_gemm_kernel", "achieved": round(achieved, 2),
                    "peak": round(alu_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / alu_peak, 4),
                    "traffic": profiled_traffic(f"svdq_int4_gemm_{w.name}.md", INT4_SOURCES),
                    "peak_note": f"fp32 rescale bound: 2 fp32 operations per output element and 64-group, "
                                 f"128 fp32 lanes x {n_sm} SMs x {sm_hz / 1e6:.0f} MHz (sampled); "
                                 f"vs FP8 tensor peak (2 x {peak_src} sustained bf16) {fp8_peak:.0f} TFLOP/s: "
                                 f"{achieved / fp8_peak:.4f}"}
    qbytes = quantize_bytes_int4(w) if int4 else quantize_bytes(w)
    q_gbs = qbytes / (k1_ms * 1e-3) / 1e9
    roofline_q = {"bound": "hbm", "kernel": "quantize_tma_kernel", "achieved": round(q_gbs, 1),
                  "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(q_gbs / peaks["hbm_gbs"], 4),
                  "traffic": None if int4 else profiled_traffic(f"quantize_tma_{w.name}.md", QUANT_SOURCES),
                  "algorithmic_bytes": qbytes}

    extras = {}
    e2e = None
    cpu = None
    if not args.no_extras and int4:
        e2e, cpu = int4_extras(args, w, step4, X, Y, X_cpu, W_cpu, flops_step, world, rank_id, timed)
    elif not args.no_extras:
        n_x = max(5, args.steps // 2)
        # fused, unfused (same arithmetic, separate passes) and no branch (rank 0)
        # interleaved step by step, so that the comparison sees the same clocks
        legs = [lambda i, ev: step(i, ev=ev), lambda i, ev: step(i, variant=S.SVDQ_UNFUSED, ev=ev)]
        if w.rank:
            legs.append(lambda i, ev: step(i, rank0=True, ev=ev))
        res = timed(n_x, lambda i, ev: [f(i, e) for f, e in zip(legs, ev)], nlegs=len(legs))
        (k1f, k2f), (k1u, k2u) = res[0], res[1]
        k1z, k2z = res[2] if w.rank else res[0]
        # bf16 cuBLAS X W^T through torch, rotating (X, W) copies the same way
        n_c = max(2, min(8, -(-2 * L2_BYTES // (X.numel() * 2 + W.numel() * 2))))
        cub_sets = [(X, W)] + [(X.clone(), W.clone()) for _ in range(n_c - 1)]

        def cublas(i, ev):
            Xc, Wc = cub_sets[i % n_c]
            ev[0].record(stream)
            torch.nn.functional.linear(Xc, Wc)
            ev[1].record(stream)
            ev[2].record(stream)
        kc, _ = timed(n_x, cublas)
        # warm L2: the same inputs every step (no rotation)
        k1w, k2w = timed(n_x, lambda i, ev: step(0, ev=ev))
        # the GEMM alone, launched back to back on the rotating inputs with one
        # pair of events around the block: its sustained duration per launch
        # (the per-kernel pass above also pays each launch's latency)
        gemm_block_ms = timed_block(n_x, lambda i: S.svdq_linear(Qx, Sx, T if w.rank else None, sets[i % n_sets][1],
                                                                  S.SVDQ_FUSED, out=Y)) / n_x
        # the quantizer alone, back to back on the rotating inputs (its launches
        # overlap as in a network; no GEMM's dirty Y to write back between them)
        quant_block_ms = timed_block(n_x, lambda i: S.svdq_quantize_act(
            sets[i % n_sets][0], sets[i % n_sets][1].inv_lam, sets[i % n_sets][1].L1p, w.rank, w.N, S.SVDQ_FUSED,
            out=(Qx, Sx, T))) / n_x
        lay = statistics.mean(step_ms)
        lay_f = statistics.mean(a + b for a, b in zip(k1f, k2f))
        q10, q50, q90 = np.percentile(step_ms, [10, 50, 90])
        extras = {
            "layer_ms_serialized": round(statistics.mean(step_ms), 4),
            "layer_ms_p10_p50_p90": [round(float(q10), 4), round(float(q50), 4), round(float(q90), 4)],
            "warm_l2_layer_ms": round(statistics.mean(a + b for a, b in zip(k1w, k2w)), 4),
            "warm_l2_quantize_ms": round(statistics.mean(k1w), 4),
            "warm_l2_gemm_ms": round(statistics.mean(k2w), 4),
            "gemm_square_rank0": square_gemm_rate(S, dev),
            "prepare_ms_offline": round(prepare_ms, 3),
            "quantize_ms": round(k1_ms, 4), "gemm_ms": round(k2_ms, 4), "layer_ms": round(ms_per_step, 4),
            "unfused_layer_ms": round(statistics.mean(a + b for a, b in zip(k1u, k2u)), 4),
            "rank0_layer_ms": round(statistics.mean(a + b for a, b in zip(k1z, k2z)), 4),
            "rank0_gemm_ms": round(statistics.mean(k2z), 4),
            "gemm_block_ms": round(gemm_block_ms, 4),
            "gemm_block_frac": round(gemm_flops(w) / (gemm_block_ms * 1e-3) / 1e12 / fp4_peak, 4),
            "gemm_block_frac_datasheet_9pf": round(gemm_flops(w) / (gemm_block_ms * 1e-3) / 1e12 / DATASHEET_FP4_TFLOPS, 4),
            "quantize_block_ms": round(quant_block_ms, 4),
            "quantize_block_gbs": round(quantize_bytes(w) / (quant_block_ms * 1e-3) / 1e9, 1),
            "quantize_block_frac_hbm": round(quantize_bytes(w) / (quant_block_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "bf16_cublas_ms": round(statistics.mean(kc), 4),
            "bf16_cublas_tflops": round(2 * w.M * w.N * w.K / (statistics.mean(kc) * 1e-3) / 1e12, 1),
        }
        extras["interleaved_fused_layer_ms"] = round(lay_f, 4)
        extras["interleaved_fused_gemm_ms"] = round(statistics.mean(k2f), 4)
        extras["lowrank_overhead_layer"] = round(lay_f / extras["rank0_layer_ms"] - 1, 4)
        extras["lowrank_overhead_gemm"] = round(statistics.mean(k2f) / extras["rank0_gemm_ms"] - 1, 4)
        extras["unfused_overhead_layer"] = round(extras["unfused_layer_ms"] / extras["rank0_layer_ms"] - 1, 4)

        # the INT4 variant (64-element groups, fp16 scales) of the same layer
        Qx4, Sx4 = int4_act_buffers()
        step4c, sets4 = make_step4(Qx4, Sx4)
        for i in range(3):
            step4c(i)
        int4_layer = timed_block(n_x, lambda i: step4c(i)) / n_x
        k1i, k2i = timed(n_x, lambda i, ev: step4c(i, ev), warm=0)
        int4_gemm_block = timed_block(n_x, lambda i: S.svdq_int4_linear(Qx4, Sx4, T, sets4[i % n_sets], out=Y)) / n_x
        S.svdq_check()
        g4 = statistics.mean(k2i)
        extras["int4"] = {
            "layer_ms": round(int4_layer, 4),
            "layer_tflops": round(flops_step / (int4_layer * 1e-3) / 1e12, 1),
            "quantize_ms": round(statistics.mean(k1i), 4),
            "gemm_ms": round(g4, 4),
            "gemm_tflops": round(gemm_flops(w) / (g4 * 1e-3) / 1e12, 1),
            "gemm_block_ms": round(int4_gemm_block, 4),
            "gemm_block_tflops": round(gemm_flops(w) / (int4_gemm_block * 1e-3) / 1e12, 1),
            "gemm_block_frac_alu": round(gemm_flops(w) / (int4_gemm_block * 1e-3) / 1e12 / alu_peak, 4),
            "gemm_block_frac_fp8": round(gemm_flops(w) / (int4_gemm_block * 1e-3) / 1e12 / fp8_peak, 4),
            "alu_peak_tflops": round(alu_peak, 1), "fp8_peak_tflops": round(fp8_peak, 1),
        }

        # the other FLUX projections, where the GEMM target is stated
        extras["other_flux_shapes"] = [flux_shape_summary(S, o, dev, n_x, fp4_peak)
                                       for o in (synth.FLUX_MLP_UP, synth.FLUX_MLP_DOWN) if o.name != w.name]

        # how the workload's groups sit in the E4M3 scale range (activations of
        # one step, the prepared weights)
        S.svdq_quantize_act(X, P.inv_lam, P.L1p, w.rank, w.N, S.SVDQ_FUSED, out=(Qx, Sx, T))
        extras["scale_groups"] = {"activations": scale_group_stats(S, Sx, w.M, w.K),
                                  "weights": scale_group_stats(S, P.Sr, w.N, w.K)}

        extras["deltaquant"] = deltaquant_summary(S, dev, n_x)
        extras["deltaquant"]["frac_hbm"] = round(extras["deltaquant"]["gbs"] / peaks["hbm_gbs"], 4)

        # end to end through the public API with host buffers: every step copies
        # its X in from pinned host memory and its Y out to pinned host memory.
        X_host = X_cpu.pin_memory()
        Y_host = [torch.empty(w.M, w.N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]

        def e2e_step(i, ev):       # one step at a time: upload, layer, download
            ev[0].record(stream)
            X.copy_(X_host, non_blocking=True)
            S.svdq_quantize_act(X, P.inv_lam, P.L1p, w.rank, w.N, S.SVDQ_FUSED, out=(Qx, Sx, T))
            S.svdq_linear(Qx, Sx, T, P, S.SVDQ_FUSED, out=Y)
            Y_host[0].copy_(Y, non_blocking=True)
            ev[1].record(stream)
            ev[2].record(stream)
        ke, _ = timed(n_x, e2e_step)
        e2e_serial_ms = aggregate_max(sum(ke), world) / n_x

        # the same, pipelined as a serving loop would run it: uploads and
        # downloads on their own streams (one copy engine per direction), two
        # device buffer sets, so step i's layer overlaps step i+1's upload and
        # step i-1's download; the timed region spans the first upload to the
        # last download
        Xd, Yd = [X, X.clone()], [Y, torch.empty_like(Y)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        up, done, down = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

        def e2e_pipelined(n):
            t_a, t_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            torch.cuda._sleep(2_000_000)
            t_a.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(n):
                b = i % 2
                if i >= 2:
                    s_in.wait_event(done[b])          # step i-2's layer has read Xd[b]
                with torch.cuda.stream(s_in):
                    Xd[b].copy_(X_host, non_blocking=True)
                up[b].record(s_in)
                stream.wait_event(up[b])
                if i >= 2:
                    stream.wait_event(down[b])        # step i-2's Y has left Yd[b]
                S.svdq_quantize_act(Xd[b], P.inv_lam, P.L1p, w.rank, w.N, S.SVDQ_FUSED, out=(Qx, Sx, T))
                S.svdq_linear(Qx, Sx, T, P, S.SVDQ_FUSED, out=Yd[b])
                done[b].record(stream)
                s_out.wait_event(done[b])
                with torch.cuda.stream(s_out):
                    Y_host[b].copy_(Yd[b], non_blocking=True)
                down[b].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            t_b.record(stream)
            torch.cuda.synchronize()
            return t_a.elapsed_time(t_b)
        e2e_pipelined(3)
        e2e_ms = aggregate_max(e2e_pipelined(n_x), world) / n_x
        e2e = {"value": round(flops_step * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2,
               "ms_per_step": round(e2e_ms, 4),
               "pipeline": "uploads and downloads on their own streams, two device buffer sets",
               "ms_per_step_one_at_a_time": round(e2e_serial_ms, 4)}
        S.svdq_check()

        if rank_id == 0 and world == 1:
            fn, fl, sample = oracle_sample(w, X_cpu, W_cpu)
            v, n, el = time_cpu(fn, fl, args.cpu_seconds)
            cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                   "sample": sample, "repeats": n, "seconds": round(el, 2), "cpu_model": cpu_model()}
            try:
                from threadpoolctl import threadpool_limits
                with threadpool_limits(limits=1):
                    v1, _, _ = time_cpu(fn, fl, max(1.0, args.cpu_seconds / 4))
                cpu["value_1_core"] = round(v1, 6)
            except Exception as e:  # the single-core figure is informative only
                cpu["value_1_core"] = f"unavailable: {type(e).__name__}"

    if rank_id == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "int4(e4m3 bytes)+bf16" if int4 else "nvfp4+bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "codec": args.codec, "M_per_gpu": w.M, "K": w.K, "N": w.N, "rank": w.rank, "alpha": w.alpha,
                       "global_tokens": w.M * world, "parallelism": f"token-parallel x{world} (weights replicated)",
                       "l2": l2_note},
            "roofline": roofline, "roofline_quantize": roofline_q,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": clocks,
            "extras": extras,
            "kernel_src": {"gemm": kernel_source_hash(GEMM_SOURCES), "quantize": kernel_source_hash(QUANT_SOURCES)},
        }
        print(json.dumps(line), flush=True)
        if args.extra_json:
            with open(args.extra_json, "a") as f:
                f.write(json.dumps(line) + "\n")
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def run_deltaquant_only(args) -> int:
    """The DeltaQuant encoder alone on one GPU (a few launches, no other kernel)."""
    from w4a4_diffusion_model_b200 import svdq as S
    if not torch.cuda.is_available():
        raise RuntimeError("the DeltaQuant encoder needs a CUDA device (there is no CPU fallback)")
    S.load()
    dev = torch.device("cuda", 0)
    print(json.dumps(deltaquant_summary(S, dev, max(1, args.steps))), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.deltaquant_only:
        return run_deltaquant_only(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
