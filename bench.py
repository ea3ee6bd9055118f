"""Benchmark of the INT8 ConvRot linear layer on B200.

One step = the seven Qwen3-VL-32B-shaped linears of one decoder layer at
M = 12 conditioning tokens (q, k, v, o, gate, up, down), each a full
ConvRot INT8 linear (activation rotation + row quantisation kernel, then the
tcgen05 INT8 GEMM with fused dequantisation) through the C ABI, with
weights already rotated, quantised and resident in HBM.  The metric is the
weight-stream bandwidth in GB/s of algorithmic bytes; the roofline object
reports the GEMM kernel against the measured HBM copy bandwidth.  A second
measurement runs the same seven linears at prefill size M = 4096 and
reports INT8 tensor TOPS against the dense INT8 peak.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 it is launched under torch.distributed.run; every rank runs an
independent replica (the layer needs no exchange between GPUs), and the
whole-job value is the bytes all ranks moved over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "ConvRot INT8 linear TOPS & weight-stream GB/s on 1 B200, % of INT8/HBM roofline"
UNIT = "GB/s"
WORKLOAD = "qwen3vl32b_layer_7linears_decode_m12"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0     # nominal dense ratio (4.5 / 2.25 PFLOP/s), a note beside the measured INT8 peak
CPU_SAMPLE_ROWS_DIV = 64  # reference arm: each step one linear with its first N/64 weight rows


# --------------------------------------------------------------------------- helpers
def linear_bytes(m: int, n: int, k: int) -> int:
    """Algorithmic HBM bytes of one ConvRot INT8 linear: weight codes and
    scales, the BF16 activations, the INT8 activations written and read
    back, their scales, and the BF16 output."""
    return n * k + 4 * n + 2 * m * k + m * k + m * k + 4 * m + 2 * m * n


def gemm_bytes(m: int, n: int, k: int) -> int:
    """Algorithmic bytes of the GEMM kernel alone."""
    return n * k + 4 * n + m * k + 4 * m + 2 * m * n


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


GEMM_SOURCES = ("common.cuh", "gemm_i8.cu", "gemm_i8.h")


def kernel_source_hash(only=None) -> str:
    """Hash of the CUDA sources (all of them, or the named files)."""
    csrc = os.path.join(ROOT, "rotated_int8_quantized_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")) and (only is None or f in only):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, if it was taken on the current sources of that kernel (the GEMM's
    files; else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.tsv")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(GEMM_SOURCES)
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.rstrip("\n").split("\t")
            if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload and parts[2] == want:
                return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms."""
    FIELDS = ("timestamp,index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, pci_bus_id: str | None):
        self.pci = (pci_bus_id or "").lower()
        self.rows = []
        self.proc = None
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.6)

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self, windows=None):
        """Stop sampling; the summary over the marked windows (or the given
        ones)."""
        if self.proc is None:
            return None
        if self.proc.poll() is None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return self.summary(self.windows if windows is None else windows)

    def summary(self, windows):
        sm, smax, reasons, n_all = [], None, set(), 0
        for t, line in self.rows:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            if self.pci and not parts[2].lower().endswith(self.pci):
                continue
            n_all += 1
            if not any(a - 0.05 <= t <= b + 0.05 for a, b in windows):
                continue
            try:
                sm.append(float(parts[3]))
                smax = float(parts[4])
            except ValueError:
                continue
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
            for name, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "samples_all": n_all}


def measure_int8_peak(device, n: int = 8192, reps: int = 10):
    """The dense INT8 tensor peak as a library reaches it on this GPU: a
    large torch._int_mm (cuBLASLt INT8 x INT8 -> INT32, A row-major, B
    column-major) of n x n x n, 2 n^3 ops, best of `reps` CUDA-event-timed
    launches after warm-up (run, not read)."""
    gen = torch.Generator(device=device).manual_seed(8)
    a = torch.randint(-127, 128, (n, n), generator=gen, device=device, dtype=torch.int32).to(torch.int8)
    b = torch.randint(-127, 128, (n, n), generator=gen, device=device, dtype=torch.int32).to(torch.int8)
    bt = b.t()
    for _ in range(3):
        torch._int_mm(a, bt)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, bt)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    ops = 2.0 * n ** 3
    del a, b, bt
    torch.cuda.empty_cache()
    return {"tops": ops / min(times) / 1e12, "median_tops": ops / statistics.median(times) / 1e12,
            "shape": [n, n, n], "how": "torch._int_mm (cuBLASLt INT8 -> INT32), best of %d, CUDA events" % reps}


# --------------------------------------------------------------------------- GPU arm
class Layer:
    """The seven quantised linears of one layer, resident on the device."""

    def __init__(self, cr, lins, device):
        self.cr = cr
        self.lins = lins
        self.w = []
        for lin in lins:
            w_bf = lin.w_torch(device)
            self.w.append(cr.quantize_weight(w_bf))
            del w_bf
        torch.cuda.synchronize()


def make_io(cr, layer, lins, device):
    xs = [lin.x_torch(device) for lin in lins]
    ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
    wss = [cr.make_workspace(lin.m, w) for lin, w in zip(lins, layer.w)]
    return xs, ys, wss


def run_step(cr, layer, xs, ys, wss, stream):
    """The layer's linears one call each (per-linear entry point)."""
    for x, w, y, ws in zip(xs, layer.w, ys, wss):
        cr.convrot_linear_int8(x, w, y, ws, stream)


def count_launches(fn, stream) -> int:
    """Kernel launches one call makes: capture it in a CUDA graph and count
    the kernel nodes."""
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.stream(stream):
        fn()                         # first call configures the kernels outside capture
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    try:
        from cuda.bindings import runtime as rt
        raw = g.raw_cuda_graph()
        handle = rt.cudaGraph_t(init_value=int(raw)) if not isinstance(raw, rt.cudaGraph_t) else raw
        err, nodes, num = rt.cudaGraphGetNodes(handle, 64)
        n = 0
        for node in nodes[:num]:
            e2, t = rt.cudaGraphNodeGetType(node)
            if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                n += 1
        return n
    except Exception as e:  # noqa: BLE001
        print("launch count unavailable: %r" % (e,), file=sys.stderr)
        return -1


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def time_region(fn, steps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3


def keep_busy(stream, us: float = 60.0):
    """Queue a short device-side spin ahead of a timed launch so that the
    host's launch overhead is not inside the CUDA-event interval."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 2000))


def gemm_batch_kernel_time(cr, layer, lins, xs, reps, stream, device):
    """Per-launch time of the batched GEMM kernel (all linears of the step in
    one launch) with CUDA events on the launching stream; the activation
    prologue runs before, untimed."""
    xqs = [torch.empty((lin.m, lin.k), dtype=torch.int8, device=device) for lin in lins]
    sxs = [torch.empty((lin.m,), dtype=torch.float32, device=device) for lin in lins]
    ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
    gb = cr.GemmBatch(xqs, sxs, layer.w, ys)
    torch.cuda.synchronize()        # the zeroed workspace is ready before `stream` uses it
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps + 2):
        keep_busy(stream)
        for x, xq, sx in zip(xs, xqs, sxs):
            cr.convrot_quantize_act(x, xq, sx, stream=stream)
        if i >= 2:
            evs[i - 2][0].record(stream)
        gb(stream)
        if i >= 2:
            evs[i - 2][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / reps / 1e3


def gemm_kernel_times(cr, layer, lins, xs, reps, stream, device):
    """Per-launch GEMM kernel time per linear with CUDA events on the
    launching stream (activation prologue launched before each, untimed)."""
    out = []
    for lin, w, x in zip(lins, layer.w, xs):
        xq = torch.empty((lin.m, lin.k), dtype=torch.int8, device=device)
        sx = torch.empty((lin.m,), dtype=torch.float32, device=device)
        y = torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device)
        ws = cr.make_workspace(lin.m, w, linear=False)
        torch.cuda.synchronize()    # the zeroed workspace is ready before `stream` uses it
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps + 2):
            keep_busy(stream)
            cr.convrot_quantize_act(x, xq, sx, stream=stream)
            if i >= 2:
                evs[i - 2][0].record(stream)
            cr.convrot_gemm_i8(xq, sx, w, y, None, ws, stream)
            if i >= 2:
                evs[i - 2][1].record(stream)
        torch.cuda.synchronize()
        t = sum(a.elapsed_time(b) for a, b in evs) / reps / 1e3
        out.append((lin, t))
    return out


def prologue_kernel_times(cr, lins, xs, reps, stream, device, l2_bytes=126 << 20):
    """Per-launch time of the activation prologue (rotation + row
    quantisation) per linear, CUDA events on the launching stream.  The
    launches cycle through enough distinct inputs and outputs (copies of the
    linear's activations) that together they exceed twice the L2, so every
    launch reads its input from HBM."""
    out = []
    for lin, x in zip(lins, xs):
        per = 3 * lin.m * lin.k
        copies = max(1, min(8, -(-2 * l2_bytes // per)))
        srcs = [x] + [x.clone() for _ in range(copies - 1)]
        xqs = [torch.empty((lin.m, lin.k), dtype=torch.int8, device=device) for _ in range(copies)]
        sxs = [torch.empty((lin.m,), dtype=torch.float32, device=device) for _ in range(copies)]
        torch.cuda.synchronize()
        for i in range(copies):
            cr.convrot_quantize_act(srcs[i], xqs[i], sxs[i], stream=stream)
        n = max(reps, 2 * copies)
        keep_busy(stream, 200.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for r in range(n):
            i = r % copies
            cr.convrot_quantize_act(srcs[i], xqs[i], sxs[i], stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        out.append((lin, e0.elapsed_time(e1) / n / 1e3, copies))
        del srcs, xqs, sxs
    torch.cuda.empty_cache()
    return out


def all_max(v: float, world: int, device="cuda") -> float:
    """The maximum of `v` over the ranks (the slowest rank's time)."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step: int, steps: int, elapsed_local: float, world: int, device="cuda"):
    """Whole-job GB/s: every rank runs the same replica, so the job moved
    world x steps x bytes_per_step bytes in the slowest rank's time."""
    elapsed = all_max(elapsed_local, world, device)
    return bytes_per_step * steps * world / elapsed / 1e9, elapsed


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def _time_calls(fn, min_seconds):
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            return el / n, n


def cpu_baseline(lins, single_seconds: float = 8.0, all_seconds: float = 4.0):
    """The oracle, as it stands (plain C), on the host cores: the decode
    layer (the seven linears at M = 12) in full against full-size weights,
    single-threaded and built with OpenMP over all cores; the tiny layer in
    full; the q matrix of the prefill layer (M = 4096), all cores in full
    when that fits in about 15 s, else a stated sample.  The weight codes of
    the timing runs are uniform random INT8 from numpy: the oracle's
    per-call work (activation rotation and quantisation, INT64 GEMM,
    dequantisation) does not depend on their values, and the offline weight
    conversion is not part of a step."""
    import oracle
    cores = host_cores()
    os.environ["OMP_NUM_THREADS"] = str(cores)
    rng = np.random.default_rng(0)
    prep = [(lin.x_np(), rng.integers(-127, 128, (lin.n, lin.k), dtype=np.int8),
             np.full(lin.n, 1e-4, np.float32)) for lin in lins]
    bytes_step = sum(linear_bytes(lin.m, lin.n, lin.k) for lin in lins)

    def decode_step():
        for x, wq, sw in prep:
            oracle.linear_int8(x, wq, sw)
    out = {"unit": UNIT, "kind": "oracle", "cores": cores}
    oracle.set_parallel(False)
    t1, n1 = _time_calls(decode_step, single_seconds)
    oracle.set_parallel(True)
    decode_step()
    ta, na = _time_calls(decode_step, all_seconds)
    out["value"] = bytes_step / ta / 1e9
    out["single_thread"] = {"value": bytes_step / t1 / 1e9, "ms_per_step": t1 * 1e3, "steps": n1, "cores": 1}
    out["all_cores"] = {"value": bytes_step / ta / 1e9, "ms_per_step": ta * 1e3, "steps": na, "cores": cores}
    # tiny layer in full (weights converted by the oracle itself)
    tl = synth.tiny()[0]
    twq, tsw = oracle.rotate_quantize(tl.w_np())
    tx = tl.x_np()
    oracle.set_parallel(False)
    tt, _ = _time_calls(lambda: oracle.linear_int8(tx, twq, tsw), 1.0)
    out["tiny_m4_k512_n256"] = {"us_per_call_single_thread": tt * 1e6,
                                "gb_s_single_thread": linear_bytes(tl.m, tl.n, tl.k) / tt / 1e9}
    # one matrix of the prefill layer: q (K = 5120, N = 8192) at M = 4096
    q = synth.qwen_layer(4096)[0]
    qwq = rng.integers(-127, 128, (q.n, q.k), dtype=np.int8)
    qsw = np.full(q.n, 1e-4, np.float32)
    macs_per_row = q.n * q.k
    rate_all = sum(12 * lin.n * lin.k for lin in lins) / ta       # MAC/s seen on the decode layer
    rows_all = q.m if q.m * macs_per_row / rate_all <= 15.0 else max(64, int(15.0 * rate_all / macs_per_row))
    oracle.set_parallel(True)
    xa = q.x_rows_np(np.arange(rows_all))
    t0 = time.perf_counter()
    oracle.linear_int8(xa, qwq, qsw)
    ta_q = (time.perf_counter() - t0) * q.m / rows_all
    oracle.set_parallel(False)
    rows_1 = 64
    x1 = q.x_rows_np(np.arange(rows_1))
    t0 = time.perf_counter()
    oracle.linear_int8(x1, qwq, qsw)
    t1_q = (time.perf_counter() - t0) * q.m / rows_1
    ops = 2 * q.m * q.n * q.k
    out["prefill_q_m4096"] = {
        "all_cores": {"tops": ops / ta_q / 1e12, "s": ta_q, "rows_timed": rows_all,
                      "extrapolated": rows_all < q.m},
        "single_thread": {"tops": ops / t1_q / 1e12, "s": t1_q, "rows_timed": rows_1, "extrapolated": True}}
    out["sample"] = ("decode layer (7 linears, M=12, full-size weights with random INT8 codes) in full: "
                     "%d single-threaded steps, %d all-core steps; tiny layer in full; prefill q at M=4096: "
                     "%d token rows on all cores, 64 single-threaded, scaled to 4096 rows"
                     % (n1, na, rows_all))
    del prep, qwq
    return out


def method_error_report():
    """What the rotation buys, computed by the oracle in FP64 on the host:
    for the tiny layer (in full), the decode layer (all 12 tokens, 256
    sampled output channels per linear) and the MiniMax qkv projection (64
    sampled tokens x 256 output channels): the relative Frobenius error
    against the unquantised FP64 product X W^T of (a) ConvRot INT8 (rotated,
    the layer built here; the BF16 output and its FP64 dequantised product)
    and (b) plain row-wise INT8 of the same X and W without rotation; and
    the activations' per-group max/RMS ratio before and after rotation."""
    import oracle
    oracle.set_parallel(True)

    def one(x_bits, w_bits):
        x = oracle.bf16_bits_to_f64(x_bits)
        w = oracle.bf16_bits_to_f64(w_bits)
        ref = oracle.matmul_nt_f64(x, w)
        nrm = float(np.linalg.norm(ref))
        wq, sw = oracle.rotate_quantize(w_bits)
        r = oracle.linear_int8(x_bits, wq, sw)
        ydq = oracle.matmul_nt_f64(r["xq"].astype(np.float64) * r["sx"][:, None].astype(np.float64),
                                   wq.astype(np.float64) * sw[:, None].astype(np.float64))
        y = oracle.bf16_bits_to_f64(r["y"])
        xq0, sx0, _ = oracle.quantize_rows(x.astype(np.float32))
        wq0, sw0, _ = oracle.quantize_rows(w.astype(np.float32))
        yu = oracle.matmul_nt_f64(xq0.astype(np.float64) * sx0[:, None].astype(np.float64),
                                  wq0.astype(np.float64) * sw0[:, None].astype(np.float64))
        yr, _ = oracle.rotate_rows(x_bits)
        g0 = x.reshape(x.shape[0], -1, 256)
        g1 = yr.astype(np.float64).reshape(x.shape[0], -1, 256)
        ratio0 = np.max(np.abs(g0), axis=2) / np.maximum(np.sqrt(np.mean(g0 ** 2, axis=2)), 1e-300)
        ratio1 = np.max(np.abs(g1), axis=2) / np.maximum(np.sqrt(np.mean(g1 ** 2, axis=2)), 1e-300)
        return {"rel_err_convrot_int8_bf16_out": float(np.linalg.norm(y - ref) / nrm),
                "rel_err_convrot_int8_dq64": float(np.linalg.norm(ydq - ref) / nrm),
                "rel_err_plain_int8_dq64": float(np.linalg.norm(yu - ref) / nrm),
                "group_max_over_rms_x": {"before_mean": float(ratio0.mean()), "before_max": float(ratio0.max()),
                                         "after_mean": float(ratio1.mean()), "after_max": float(ratio1.max())}}
    rep = {}
    t = synth.tiny()[0]
    rep["tiny"] = one(t.x_np(), t.w_np())
    rng = np.random.default_rng(5)
    dec = {}
    for lin in synth.qwen_layer(12):
        rows = np.sort(rng.choice(lin.n, 256, replace=False))
        dec[lin.name] = one(lin.x_np(), lin.w_rows_np(rows))
    rep["qwen_decode_m12"] = dec
    mm = synth.minimax_qkv(8192)[0]
    rep["minimax_qkv"] = one(mm.x_rows_np(np.sort(rng.choice(mm.m, 64, replace=False))),
                             mm.w_rows_np(np.sort(rng.choice(mm.n, 256, replace=False))))
    rep["sample"] = ("tiny in full; decode: all 12 tokens x 256 random output channels per linear; "
                     "MiniMax qkv: 64 random tokens x 256 random output channels")
    oracle.set_parallel(False)
    return rep


def prefill_secondary(cr, layer, device, stream, peaks, steps=20, warmup=3):
    """The same seven linears at M = 4096 (same weights): TOPS vs the dense
    INT8 peak measured on this GPU (a large library INT8 GEMM)."""
    lins = synth.qwen_layer(4096)
    xs = [lin.x_torch(device) for lin in lins]
    ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
    batch = cr.LinearBatch(xs, layer.w, ys)
    torch.cuda.synchronize()        # inputs and the zeroed workspace are ready before `stream` uses them
    fn = lambda: batch(stream)  # noqa: E731
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    keep_busy(stream)
    t = time_region(fn, steps, stream) / steps
    ops = sum(2 * lin.m * lin.n * lin.k for lin in lins)
    g = gemm_kernel_times(cr, layer, lins, xs, 10, stream, device)
    gops = sum(2 * lin.m * lin.n * lin.k for lin, _ in g)
    gt = sum(tt for _, tt in g)
    peak = peaks["int8_tops"]
    pro = prologue_kernel_times(cr, lins, xs, 10, stream, device)
    del batch
    # as the model feeds the layer: q, k, v read one input and gate, up
    # another, so their rotation and quantisation run once per input
    groups = {"q": "attn", "k": "attn", "v": "attn", "o": "o", "gate": "mlp", "up": "mlp", "down": "down"}
    first = {}
    for lin, x in zip(lins, xs):
        first.setdefault(groups[lin.name], x)
    shared = cr.LinearBatch([first[groups[lin.name]] for lin in lins], layer.w, ys)
    torch.cuda.synchronize()
    fn = lambda: shared(stream)  # noqa: E731
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    keep_busy(stream)
    t_shared = time_region(fn, steps, stream) / steps
    del xs, ys, shared, first
    torch.cuda.empty_cache()
    return {"workload": "qwen3vl32b_layer_7linears_prefill_m4096", "metric": "INT8 TOPS (2MNK)",
            "layer_tops": ops / t / 1e12, "ms_per_step": t * 1e3,
            "shared_inputs": {"distinct_inputs": 4, "layer_tops": ops / t_shared / 1e12,
                              "ms_per_step": t_shared * 1e3},
            "gemm_tops": gops / gt / 1e12,
            "roofline": {"bound": "tensor", "achieved": gops / gt / 1e12, "peak": peak, "unit": "TOP/s",
                         "frac": gops / gt / 1e12 / peak, "peak_source": peaks["int8_source"],
                         "frac_of_bf16_x2": gops / gt / 1e12 / (peaks["bf16_tflops"] * INT8_OVER_BF16)},
            "per_linear_gemm_tops": {lin.name: 2 * lin.m * lin.n * lin.k / tt / 1e12 for lin, tt in g},
            "prologue": {"bytes": "2MK read + MK + 4M written",
                         "timing": "launches cycle through distinct copies of the input (> 2x L2 together)",
                         "per_linear_us": {lin.name: tt * 1e6 for lin, tt, _ in pro},
                         "per_linear_gbs": {lin.name: (3 * lin.m * lin.k + 4 * lin.m) / tt / 1e9
                                            for lin, tt, _ in pro},
                         "per_linear_frac_of_hbm": {lin.name: (3 * lin.m * lin.k + 4 * lin.m) / tt / 1e9
                                                    / peaks["hbm_gbs"] for lin, tt, _ in pro},
                         "copies": {lin.name: c for lin, _, c in pro},
                         "layer_us": sum(tt for _, tt, _ in pro) * 1e6}}


def shared_input_secondary(cr, layer, lins, device, stream, peaks, steps=2000, warmup=20):
    """The decode layer as the model feeds it: q, k and v read one input,
    gate and up another (their rotation runs once), o and down their own.
    Algorithmic bytes count each distinct input once."""
    groups = {"q": "attn", "k": "attn", "v": "attn", "o": "o", "gate": "mlp", "up": "mlp", "down": "down"}
    src = {}
    for lin in lins:
        src.setdefault(groups[lin.name], lin)
    xin = {g: l.x_torch(device) for g, l in src.items()}
    xs = [xin[groups[lin.name]] for lin in lins]
    ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
    batch = cr.LinearBatch(xs, layer.w, ys)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        batch(stream)
    torch.cuda.synchronize()
    g = capture(lambda: batch(stream), stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        t = time_region(g.replay, steps, stream) / steps
    m = lins[0].m
    nbytes = sum(lin.n * lin.k + 4 * lin.n + m * lin.k + 2 * m * lin.n for lin in lins)   # weights, xq reads, y
    nbytes += sum(2 * m * l.k + m * l.k + 4 * m for l in src.values())                      # one prologue per input
    del g, batch
    return {"workload": "qwen3vl32b_layer_shared_inputs_decode_m12", "distinct_inputs": len(src),
            "gb_s": nbytes / t / 1e9, "us_per_step": t * 1e6,
            "frac_of_measured_hbm": nbytes / t / 1e9 / peaks["hbm_gbs"]}


def w4a8_secondary(cr, lins, device, stream, peaks, steps=2000, warmup=20):
    """The decode layer with INT4 ConvRot weights (W4A8): the same seven
    linears at M = 12, half the weight bytes, one batched call per step."""
    ws4, keep = [], []
    for lin in lins:
        w_bf = lin.w_torch(device)
        ws4.append(cr.quantize_weight4(w_bf))
        del w_bf
    xs = [lin.x_torch(device) for lin in lins]
    ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
    batch = cr.LinearBatchW4(xs, ws4, ys)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        batch(stream)
    torch.cuda.synchronize()
    g = capture(lambda: batch(stream), stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        t = time_region(g.replay, steps, stream) / steps
    m = lins[0].m
    nbytes = sum(lin.n * lin.k // 2 + 4 * lin.n + 2 * m * lin.k + 2 * m * lin.k + 4 * m + 2 * m * lin.n for lin in lins)
    del g, batch
    # the same INT4 weights at prefill size (M = 4096): tensor-bound
    pl = synth.qwen_layer(4096)
    pxs = [lin.x_torch(device) for lin in pl]
    pys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in pl]
    pbatch = cr.LinearBatchW4(pxs, ws4, pys)
    torch.cuda.synchronize()
    for _ in range(3):
        pbatch(stream)
    torch.cuda.synchronize()
    keep_busy(stream)
    tp = time_region(lambda: pbatch(stream), 10, stream) / 10
    pops = sum(2 * lin.m * lin.n * lin.k for lin in pl)
    del pbatch, pxs, pys, ws4
    torch.cuda.empty_cache()
    return {"workload": "qwen3vl32b_layer_7linears_decode_m12_w4a8", "int4_weight_bytes": sum(l.n * l.k // 2 for l in lins),
            "gb_s": nbytes / t / 1e9, "us_per_step": t * 1e6,
            "frac_of_measured_hbm": nbytes / t / 1e9 / peaks["hbm_gbs"],
            "weight_stream_gb_s_int8_equivalent": sum(l.n * l.k for l in lins) / t / 1e9,
            "prefill_m4096": {"layer_tops": pops / tp / 1e12, "ms_per_step": tp * 1e3,
                              "frac_of_int8_peak": pops / tp / 1e12 / peaks["int8_tops"]}}


def conv_secondary(cr, device, stream, peaks, steps=10, warmup=3):
    """VAE-decoder-shaped 3x3 convolutions (int8_convrot): NHWC BF16 in and
    out, im2col rows gathered by the prologue, INT8 GEMM; TOPS (2MNK)."""
    out = {}
    peak = peaks["int8_tops"]
    for (h, c) in ((128, 512), (256, 256)):
        seed = 77 + c
        x = synth.Linear("conv_x", h * h, c, 1, seed, None).x_torch(device).view(1, h, h, c)
        w_rows = synth.Linear("conv_w", 1, 9 * c, c, seed, None).w_torch(device)
        w_oihw = w_rows.view(c, c, 3, 3)
        wq = cr.quantize_conv_weight(w_oihw)
        y = torch.empty((1, h, h, c), dtype=torch.bfloat16, device=device)
        g = cr.conv2d_geometry(x.shape, 3, 3, 1, 1, 1)
        need = int(cr.load_library().convrot_conv2d_workspace_bytes(ctypes_byref(g), ctypes_byref(wq.handle)))
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        torch.cuda.synchronize()
        fn = lambda: cr.conv2d_int8(x, wq, 3, 3, 1, 1, 1, y=y, ws=ws, stream=stream)  # noqa: E731
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                fn()
        torch.cuda.synchronize()
        keep_busy(stream, 200.0)
        t = time_region(fn, steps, stream) / steps
        ops = 2 * (h * h) * c * (9 * c)
        out["h%d_c%d" % (h, c)] = {"ms": t * 1e3, "tops": ops / t / 1e12, "frac_of_int8_ref": ops / t / 1e12 / peak,
                                   "m": h * h, "n": c, "k": 9 * c}
        del x, w_rows, w_oihw, wq, y, ws
        torch.cuda.empty_cache()
    out["workload"] = "vae_decoder_conv3x3_nhwc"
    return out


def ctypes_byref(obj):
    import ctypes
    return ctypes.byref(obj)


def minimax_secondary(cr, device, stream, peaks, steps=10, warmup=3):
    """MiniMax-H3-shaped qkv projection (K = 5376, N = 16128) at M = 8192 and
    32768 video tokens through the single-linear entry point: INT8 TOPS."""
    out = {"workload": "minimax_h3_qkv_k5376_n16128", "metric": "INT8 TOPS (2MNK)"}
    w = None
    peak = peaks["int8_tops"]
    for m in (8192, 32768):
        lin = synth.minimax_qkv(m)[0]
        if w is None:
            w_bf = lin.w_torch(device)
            w = cr.quantize_weight(w_bf)
            del w_bf
        x = lin.x_torch(device)
        y = torch.empty((m, lin.n), dtype=torch.bfloat16, device=device)
        ws = cr.make_workspace(m, w)
        torch.cuda.synchronize()
        fn = lambda: cr.convrot_linear_int8(x, w, y, ws, stream)  # noqa: E731
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        keep_busy(stream)
        t = time_region(fn, steps, stream) / steps
        g = gemm_kernel_times(cr, _OneWeight(w), [lin], [x], 10, stream, device)[0][1]
        ops = 2 * m * lin.n * lin.k
        out["m%d" % m] = {"linear_tops": ops / t / 1e12, "ms": t * 1e3, "gemm_tops": ops / g / 1e12,
                          "gemm_frac": ops / g / 1e12 / peak, "gemm_ms": g * 1e3}
        del x, y, ws
        torch.cuda.empty_cache()
    out["peak"] = peak
    return out


class _OneWeight:
    def __init__(self, w):
        self.w = [w]


def stack_secondary(cr, device, stream, peaks, layers=50, steps=5, warmup=2):
    """The 50-layer stack of the seven Qwen linears (350 INT8 weights,
    24.4 GB resident) run back to back, one batched call per layer, at
    M = 12 and M = 512 (one CUDA graph per pass): weight-stream GB/s."""
    lins12 = synth.qwen_stack(12, layers)
    t0 = time.time()
    ws = []
    for lin in lins12:
        w_bf = lin.w_torch(device)
        ws.append(cr.quantize_weight(w_bf))
        del w_bf
    torch.cuda.synchronize()
    out = {"workload": "qwen3vl32b_stack_%dlayers" % layers, "weights": len(ws),
           "weight_gb": sum(lin.n * lin.k for lin in lins12) / 1e9, "setup_s": time.time() - t0}
    for m in (12, 512):
        lins = synth.qwen_stack(m, layers)
        xs = [lin.x_torch(device) for lin in lins]
        ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
        batches = [cr.LinearBatch(xs[7 * i:7 * i + 7], ws[7 * i:7 * i + 7], ys[7 * i:7 * i + 7])
                   for i in range(layers)]
        torch.cuda.synchronize()

        def one_pass():
            for b in batches:
                b(stream)
        with torch.cuda.stream(stream):
            one_pass()
        torch.cuda.synchronize()
        launches_per_layer = count_launches(lambda: batches[0](stream), stream)
        g = capture(one_pass, stream)
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                g.replay()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):     # replay() launches on the current stream
            t = time_region(g.replay, steps, stream) / steps
        nbytes = sum(linear_bytes(lin.m, lin.n, lin.k) for lin in lins)
        ops = sum(2 * lin.m * lin.n * lin.k for lin in lins)
        out["m%d" % m] = {"gb_s": nbytes / t / 1e9, "ms_per_pass": t * 1e3, "tops": ops / t / 1e12,
                          "frac_of_measured_hbm": nbytes / t / 1e9 / peaks["hbm_gbs"],
                          "launches_per_pass": launches_per_layer * layers if launches_per_layer > 0 else None}
        del g, batches, xs, ys
        torch.cuda.empty_cache()
    del ws
    torch.cuda.empty_cache()
    return out


def run_profile(args):
    """A few plain (eager) steps of one workload for an ncu capture: no
    timing, no JSON.  Weight generation and quantisation run first."""
    import rotated_int8_quantized_b200 as cr
    cr.load_library()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    if args.profile == "conv":
        # the VAE-decoder-shaped 3x3 convolution, 256 x 256 x 256 -> 256
        h, c = 256, 256
        x = synth.Linear("conv_x", h * h, c, 1, 77 + c, None).x_torch(device).view(1, h, h, c)
        w = synth.Linear("conv_w", 1, 9 * c, c, 77 + c, None).w_torch(device).view(c, c, 3, 3)
        wq = cr.quantize_conv_weight(w)
        torch.cuda.synchronize()
        for _ in range(args.steps):
            cr.conv2d_int8(x, wq, 3, 3, 1, 1, 1)
        torch.cuda.synchronize()
        cr.convrot_device_status()
        print("profile run ok: conv, %d steps" % args.steps)
        return
    if args.profile == "w4a8":
        # the decode layer with INT4 weights (seven weight conversions, then
        # the W4A8 steps)
        lins = synth.qwen_layer(12)
        ws4 = []
        for lin in lins:
            w_bf = lin.w_torch(device)
            ws4.append(cr.quantize_weight4(w_bf))
            del w_bf
        xs = [lin.x_torch(device) for lin in lins]
        ys = [torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=device) for lin in lins]
        batch = cr.LinearBatchW4(xs, ws4, ys)
        torch.cuda.synchronize()
        for _ in range(args.steps):
            batch()
        torch.cuda.synchronize()
        cr.convrot_device_status()
        print("profile run ok: w4a8, %d steps" % args.steps)
        return
    if args.profile == "m512":
        # one layer of the 50-layer stack at M = 512
        lins = synth.qwen_stack(512, layers=1)
    else:
        lins = synth.qwen_layer({"decode": 12, "prefill": 4096}[args.profile])
    layer = Layer(cr, lins, device)
    xs, ys, wss = make_io(cr, layer, lins, device)
    stream = torch.cuda.current_stream()
    batch = cr.LinearBatch(xs, layer.w, ys)
    torch.cuda.synchronize()
    for _ in range(args.steps):
        batch(stream)
    torch.cuda.synchronize()
    cr.convrot_device_status(stream)
    print("profile run ok: %s, %d steps" % (args.profile, args.steps))


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    import rotated_int8_quantized_b200 as cr
    cr.load_library()
    peaks, peak_kind = load_peaks()

    try:
        pr = torch.cuda.get_device_properties(device)
        pci = "%02x:%02x.0" % (int(pr.pci_bus_id), int(pr.pci_device_id))
    except Exception:
        pci = None
    clocks = ClockSampler(pci)
    clocks.start()
    w0 = time.time()
    int8_peak = measure_int8_peak(device)
    int8_window = (w0, time.time())
    peaks["int8_tops"] = int8_peak["tops"]
    peaks["int8_source"] = "measured"

    lins = synth.qwen_layer(12)
    layer = Layer(cr, lins, device)
    xs, ys, wss = make_io(cr, layer, lins, device)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()

    batch = cr.LinearBatch(xs, layer.w, ys)
    torch.cuda.synchronize()        # the zeroed workspace is ready before `stream` uses it
    launches_per_step = count_launches(lambda: batch(stream), stream)
    fn_eager = lambda: batch(stream)  # noqa: E731
    with torch.cuda.stream(stream):
        fn_eager()                      # first call configures kernels (outside capture)
        run_step(cr, layer, xs, ys, wss, stream)
    torch.cuda.synchronize()
    graph = capture(fn_eager, stream) if not args.no_graph else None
    step = (lambda: graph.replay()) if graph is not None else fn_eager

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    cr.convrot_device_status(stream)

    barrier(world)
    torch.cuda.synchronize()
    w0 = time.time()
    with torch.cuda.stream(stream):
        elapsed = time_region(step, args.steps, stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    barrier(world)
    bytes_step = sum(linear_bytes(lin.m, lin.n, lin.k) for lin in lins)
    value, elapsed = job_throughput(bytes_step, args.steps, elapsed, world)
    cr.convrot_device_status(stream)

    # the same layer through the per-linear entry point (14 launches), for context
    graph1 = capture(lambda: run_step(cr, layer, xs, ys, wss, stream), stream) if not args.no_graph else None
    step1 = (lambda: graph1.replay()) if graph1 is not None else (lambda: run_step(cr, layer, xs, ys, wss, stream))
    with torch.cuda.stream(stream):
        for _ in range(3):
            step1()
        torch.cuda.synchronize()
        per_linear_t = time_region(step1, max(10, args.steps // 4), stream) / max(10, args.steps // 4)
    del graph1

    # dominant kernel: the batched GEMM (one launch over the 7 weights), CUDA
    # events on the launching stream around each launch
    gt = gemm_batch_kernel_time(cr, layer, lins, xs, 50, stream, device)
    gb = sum(gemm_bytes(lin.m, lin.n, lin.k) for lin in lins)
    achieved = gb / gt / 1e9
    g1 = gemm_kernel_times(cr, layer, lins, xs, 10, stream, device)
    traffic = profiled_traffic("gemm_i8_tc_kernel", WORKLOAD)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "kernel": "gemm_i8_tc_kernel (one launch over the 7 weights)", "peak_source": peak_kind,
                "bytes_per_launch": gb, "us_per_launch": gt * 1e6,
                "single_linear_launch_gbs": {lin.name: gemm_bytes(lin.m, lin.n, lin.k) / t / 1e9
                                             for lin, t in g1}}

    # end to end through the C ABI from pinned host buffers: the step's seven
    # inputs sit in one pinned slab (one host-to-device copy) and its seven
    # outputs land in one (one device-to-host copy).  Serving streams steps:
    # two sets of device buffers, the copies on their own streams, so step
    # i + 1's inputs go up and step i - 1's outputs come down while step i
    # computes; every step still moves its own inputs and outputs inside the
    # timed region.  The serial variant (copy, compute, copy on one stream)
    # is reported beside it.
    x_sizes = [lin.m * lin.k for lin in lins]
    y_sizes = [lin.m * lin.n for lin in lins]
    dxs = [torch.empty(sum(x_sizes), dtype=torch.bfloat16, device=device) for _ in range(2)]
    dys = [torch.empty(sum(y_sizes), dtype=torch.bfloat16, device=device) for _ in range(2)]
    batches_e = []
    for dx, dy in zip(dxs, dys):
        xs_e = [v.view(lin.m, lin.k) for v, lin in zip(torch.split(dx, x_sizes), lins)]
        ys_e = [v.view(lin.m, lin.n) for v, lin in zip(torch.split(dy, y_sizes), lins)]
        for src, dst in zip(xs, xs_e):
            dst.copy_(src)
        batches_e.append(cr.LinearBatch(xs_e, layer.w, ys_e))
    hx = dxs[0].cpu().pin_memory()
    hys = [torch.empty(dys[0].shape, dtype=dys[0].dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize()
    for b in range(2):                      # every event recorded once before the first wait
        comp_done[b].record(stream)
        out_done[b].record(stream)
    state = {"i": 0}

    def e2e_step():
        b = state["i"] & 1
        state["i"] += 1
        s_in.wait_event(comp_done[b])       # step i - 2 has read dxs[b]
        with torch.cuda.stream(s_in):
            dxs[b].copy_(hx, non_blocking=True)
        in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        stream.wait_event(out_done[b])      # step i - 2's outputs have left dys[b]
        batches_e[b](stream)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            hys[b].copy_(dys[b], non_blocking=True)
        out_done[b].record(s_out)

    def e2e_region(steps):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(steps):
            e2e_step()
        for b in range(2):
            stream.wait_event(out_done[b])
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end) / 1e3

    def serial_step():
        dxs[0].copy_(hx, non_blocking=True)
        batches_e[0](stream)
        hys[0].copy_(dys[0], non_blocking=True)

    e2e_steps = max(10, min(args.steps, 500))
    with torch.cuda.stream(stream):
        for _ in range(4):
            e2e_step()
        torch.cuda.synchronize()
        w1 = time.time()
        e2e_t = e2e_region(e2e_steps)
        clocks.mark(w1, time.time())
        for _ in range(3):
            serial_step()
        torch.cuda.synchronize()
        serial_t = time_region(serial_step, e2e_steps, stream)
    e2e_value, e2e_t = job_throughput(bytes_step, e2e_steps, e2e_t, world)
    serial_value, serial_t = job_throughput(bytes_step, e2e_steps, serial_t, world)
    # the sampler keeps running through the secondary measurements, each
    # summarised over its own window below
    clk = clocks.summary(clocks.windows) if clocks.proc is not None else None
    if clk is not None:
        int8_peak["clocks"] = clocks.summary([int8_window])
    sec_windows = {}
    h2d = sum(2 * lin.m * lin.k for lin in lins)
    d2h = sum(2 * lin.m * lin.n for lin in lins)
    e2e = {"value": e2e_value, "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "us_per_step": e2e_t / e2e_steps * 1e6, "pipelining": "double-buffered: copies on two streams overlap the "
                                                                 "neighbouring steps' compute",
           "serial": {"value": serial_value, "us_per_step": serial_t / e2e_steps * 1e6}}
    del batches_e, dxs, dys, dx, dy, xs_e, ys_e, hx, hys

    def timed_window(name, fn):
        t0 = time.time()
        r = fn()
        sec_windows[name] = (t0, time.time())
        return r

    secondary = None
    if not args.no_prefill:
        secondary = timed_window("prefill", lambda: prefill_secondary(cr, layer, device, stream, peaks))
    cr.convrot_device_status(stream)
    others = {"shared_inputs": shared_input_secondary(cr, layer, lins, device, stream, peaks),
              "w4a8": timed_window("w4a8", lambda: w4a8_secondary(cr, lins, device, stream, peaks))}
    others["conv"] = timed_window("conv", lambda: conv_secondary(cr, device, stream, peaks))
    if not args.no_minimax:
        others["minimax_qkv"] = timed_window("minimax_qkv", lambda: minimax_secondary(cr, device, stream, peaks))
        cr.convrot_device_status(stream)
    if not args.no_stack:
        del layer, xs, ys, wss, batch
        torch.cuda.empty_cache()
        others["stack"] = timed_window("stack", lambda: stack_secondary(cr, device, stream, peaks))
        cr.convrot_device_status(stream)
    secondary_clocks = None
    if clocks.proc is not None:
        clocks.stop()
        # clocks over each secondary measurement (its whole duration, set-up included)
        secondary_clocks = {name: clocks.summary([w]) for name, w in sec_windows.items()}

    cpu = None
    method_error = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(lins)
        method_error = method_error_report()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": 12,
                       "linears": [[lin.name, lin.k, lin.n] for lin in lins],
                       "weight_bytes_per_step": sum(lin.n * lin.k for lin in lins),
                       "algorithmic_bytes_per_step": bytes_step,
                       "l2": "inputs larger than L2: %.1f MB of INT8 weights streamed per step vs 126 MB L2"
                             % (sum(lin.n * lin.k for lin in lins) / 1e6),
                       "cuda_graph": graph is not None, "entry_point": "convrot_linear_int8_batch",
                       "parallelism": "replicas" if world > 1 else "single"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clk,
            "per_linear_entry_point": {"ms_per_step": per_linear_t * 1e3,
                                       "value": bytes_step / per_linear_t / 1e9,
                                       "launches_per_step": 2 * len(lins)},
            "secondary": secondary, "more": others or None, "secondary_clocks": secondary_clocks,
            "method_error": method_error,
            "int8_peak": int8_peak, "library_build_id": cr.build_id(), "kernel_sources": kernel_source_hash(),
            "gemm_sources": kernel_source_hash(GEMM_SOURCES),
        }
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle (plain single-threaded C on the host) on the same workload:
    each step is one linear of the layer (cycling q, k, v, o, gate, up, down)
    at M = 12 with its first N/64 weight rows."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    lins = synth.qwen_layer(12)
    prepared = []
    for lin in lins:
        ns = max(1, math.ceil(lin.n / CPU_SAMPLE_ROWS_DIV))
        wq, sw = oracle.rotate_quantize(lin.w_rows_np(np.arange(ns)))
        prepared.append((lin, ns, lin.x_np(), wq, sw))
    for s in range(args.warmup):
        lin, ns, x, wq, sw = prepared[s % 7]
        oracle.linear_int8(x, wq, sw)
    nbytes = 0
    t0 = time.perf_counter()
    for s in range(args.steps):
        lin, ns, x, wq, sw = prepared[s % 7]
        oracle.linear_int8(x, wq, sw)
        nbytes += linear_bytes(lin.m, ns, lin.k)
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    sample = ("each step one linear of the layer in turn at M=12 with its first N/%d weight rows; "
              "%d steps, %.1f s" % (CPU_SAMPLE_ROWS_DIV, args.steps, el))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / max(args.steps, 1) * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": 12}, "gpu_launches": 0,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-minimax", action="store_true", help="skip the MiniMax qkv TOPS measurement")
    ap.add_argument("--no-stack", action="store_true", help="skip the 50-layer stack measurement")
    ap.add_argument("--profile", choices=["decode", "prefill", "conv", "w4a8", "m512"], default=None,
                    help="run a few eager steps of one workload for ncu (no timing)")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
