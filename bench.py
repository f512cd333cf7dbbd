"""Throughput of the sparse gated FFN forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME] [--no-cpu-baseline] [--no-extra]

One step = one pass of the whole sparse path over one batch of M tokens:
twell_gate_pack (reset + tcgen05 gate GEMM with the ReLU/TwELL/overflow
epilogue), twell_ffn_fwd (fused sparse up+down kernel, then the dense-row
overflow GEMMs) and one device-to-host read of the overflow count and the
device flags, which the host checks after the step (a count above the
dense-row capacity would make the caller retry with a larger buffer), inputs
resident in HBM.  The L2 (126 MB) is flushed with a 256 MiB write before
every timed step; the flush is outside the timed events.

The headline workload is the largest single-GPU configuration at 99%
sparsity (M=16384, K=2560, N=10240); the M=2048 and M=8192 workloads are
timed the same way and reported under "other_workloads".  Small batches
(M=16 and M=64 rows, K=2048, N=8192, 99% sparsity) are reported under
"small_batch": there every step is replayed from a CUDA graph (the launch
path of a decode loop) and four copies of the weights (4 x 100 MB, more than
L2) are used in turn, so no step finds its weights in L2.

For N > 1 (torchrun, one rank per GPU) every rank runs its own batch of the
same workload: the forward pass is token-parallel and needs no collective
("replicas only", weak scaling); times are the max over ranks.

--impl reference times the fp64 CPU oracle (the test oracle, unchanged) on the
host cores for the same workload and metric, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from activation_sparse_gated_tma_b200 import workloads as wl  # noqa: E402

METRIC = "sparse FFN fwd tokens/s @99% sparsity, % of roofline, speedup vs own dense FFN"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILES = os.path.join(ROOT, "profiles")
# Timed next to the headline workload and reported under "other_workloads".
EXTRA_WORKLOADS = ("m2048_k1536_n4096_p99_lognormal05", "m8192_k2048_n5632_loguniform_lognormal07")
FLUSH_BYTES = 256 << 20
# Small-batch workloads, timed from CUDA graphs over rotating weight copies.
SMALL_BATCH_WORKLOADS = ("sweep_m16_k2048_n8192_p99", "sweep_m64_k2048_n8192_p99")
SMALL_BATCH_COPIES = 4
# Backward pass over the hybrid activations (training), timed on these.
BACKWARD_WORKLOADS = ("m16384_k2560_n10240_p99_boost3pct", "m2048_k1536_n4096_p99_lognormal05")


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# The sources each profiled kernel is built from (its launch configuration
# lives in twell_api.cu, so that file counts for every kernel).
KERNEL_SOURCES = {
    "twell_updown": ("sparse_updown.cuh", "ptx.cuh", "twell_api.cu"),
    "gate_twell_gemm": ("tc_gemm.cuh", "epilogues.cuh", "gemm_kernels.cu", "internal.h", "ptx.cuh", "twell_api.cu"),
    "overflow_up_gemm": ("tc_gemm.cuh", "epilogues.cuh", "gemm_kernels.cu", "internal.h", "ptx.cuh", "twell_api.cu"),
    "overflow_down_gemm": ("tc_gemm.cuh", "epilogues.cuh", "gemm_kernels.cu", "internal.h", "ptx.cuh", "twell_api.cu"),
}


def kernel_source_hash(kernel: str = "") -> str:
    """Hash of the CUDA sources of `kernel` (all sources if unknown); a profile
    taken on other sources is stale."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "activation_sparse_gated_tma_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc))
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from a committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(PROFILES, f"{kernel}__{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash(kernel):
        return None
    return float(m_bytes.group(1))


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7], "sw_power": parts[8]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load)}


# ----------------------------------------------------------------------------- helpers
def workload_stats(tw, w, T, C):
    counts = tw.counts.cpu().numpy().view(np.uint16).astype(np.int64)
    per_tok = counts.sum(1)
    ov = counts > C
    return {
        "active_fraction": float(per_tok.sum() / (w.M * w.N)),
        "nnz_per_token_mean": float(per_tok.mean()),
        "nnz_per_token_p50": float(np.percentile(per_tok, 50)),
        "nnz_per_token_p99": float(np.percentile(per_tok, 99)),
        "nnz_per_token_max": int(per_tok.max()),
        "overflow_rows": int(ov.any(1).sum()),
        "overflow_tiles": int(ov.sum()),
        "twell_entries": int(np.where(ov, 0, counts).sum()),
    }


def unique_active_units(tw, C, T):
    """Number of distinct hidden units read by the fused kernel (non-overflow entries)."""
    counts = tw.counts.cpu().numpy().view(np.uint16).astype(np.int64)
    idx = tw.idx.cpu().numpy().astype(np.int64)
    M, NT = counts.shape
    used = (np.arange(C)[None, None, :] < np.minimum(counts, C)[:, :, None]) & (counts <= C)[:, :, None]
    t_i = np.broadcast_to(np.arange(NT)[None, :, None], idx.shape)
    n = (t_i * T + idx)[used]
    return int(np.unique(n).size)


def cpu_oracle_rate(d, w, rows_target_s: float, min_rows: int = 8):
    """Time the fp64 oracle's sparse forward (gate, TwELL pack, sparse y) on a
    bounded row sample; returns (tokens/s, rows, seconds, threads)."""
    import oracle
    nthreads = oracle.default_threads()
    probe = wl.subsample_rows(w.M, max(min_rows, nthreads), seed=5)
    t0 = time.perf_counter()
    oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C, rows=probe, nthreads=nthreads)
    dt = time.perf_counter() - t0
    per_row = dt / probe.size
    n = int(max(min_rows, min(w.M, rows_target_s / max(per_row, 1e-9))))
    n = max(nthreads, (n // nthreads) * nthreads) if n >= nthreads else n
    rows = wl.subsample_rows(w.M, n, seed=6)
    t0 = time.perf_counter()
    oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C, rows=rows, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return rows.size / dt, int(rows.size), dt, nthreads


def cpu_dense_oracle_rate(d, w, rows: int = 32):
    """Time the fp64 oracle's dense FFN (every hidden unit) on a small row
    sample; returns (tokens/s, rows, seconds)."""
    import oracle
    sample = wl.subsample_rows(w.M, min(rows, w.M), seed=8)
    t0 = time.perf_counter()
    oracle.ffn_dense(d["x"], d["wg_t"], d["wu_t"], d["wd"], rows=sample)
    dt = time.perf_counter() - t0
    return sample.size / dt, int(sample.size), dt


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(values, world: int, device=None):
    """Element-wise maximum of per-rank timings over all ranks (one all-reduce;
    every rank must call it).  With one rank the values come back unchanged."""
    values = [float(v) for v in values]
    if world <= 1:
        return values
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world: int, rows_per_rank: int, ms: float) -> float:
    """Tokens/s of the whole job: every rank's rows over the slowest rank's time."""
    return world * rows_per_rank / (ms * 1e-3)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    d = wl.generate(w)
    import oracle
    nthreads = oracle.default_threads()
    # Size one step to about 2 s of CPU work so --steps K --warmup W ends in minutes.
    probe = wl.subsample_rows(w.M, max(8, nthreads), seed=5)
    t0 = time.perf_counter()
    oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C, rows=probe, nthreads=nthreads)
    per_row = (time.perf_counter() - t0) / probe.size
    rows_per_step = int(min(w.M, max(nthreads, 2.0 / max(per_row, 1e-9))))
    times = []
    for i in range(args.warmup + args.steps):
        rows = wl.subsample_rows(w.M, rows_per_step, seed=100 + i)
        t0 = time.perf_counter()
        oracle.forward(d["x"], d["wg_t"], d["wu_t"], d["wd"], w.T, w.C, rows=rows, nthreads=nthreads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = rows_per_step / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "T": w.T, "C": w.C,
                   "rows_per_step": rows_per_step},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"{rows_per_step} seeded rows of {w.M} per step: fp64 gate, TwELL pack, sparse y"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- native arm
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def path_roofline(M, K, N, T, C, U, R, peaks, ms, entries=None):
    """The path roofline as the scope table's measurement rule states it:
    T_roof = max(2MKN / P_tc, B_alg / BW_hbm) with
    B_alg = 2KN + 4K*U + 2MK + 4MK + 2*M*(N/T)*(2+3C) + 4*R*N
    (W_g once; the unique W_u, W_d rows; x; y in fp32; TwELL written and read
    with bf16 values; the bf16 dense-row backup written and read)."""
    NT = N // T
    flops = 2.0 * M * K * N
    b_alg = 2.0 * K * N + 4.0 * K * U + 2.0 * M * K + 4.0 * M * K + 2.0 * M * NT * (2 + 3 * C) + 4.0 * R * N
    # The library stores TwELL values and the dense-row gates in fp32: 5 bytes per slot, 4 per gate.
    b_build = 2.0 * K * N + 4.0 * K * U + 2.0 * M * K + 4.0 * M * K + 2.0 * M * NT * (2 + 5 * C) + 8.0 * R * N
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = b_alg / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_tc, t_hbm)
    # Reported, not the target: the fp32 ALU time of the sparse products (one
    # FMA per (entry, k) for each of the dot and the axpy: 4K FLOP per listed
    # entry) against B200's fp32 FMA rate (148 SMs x 128 lanes x 2 FLOP at
    # 1965 MHz = 74.4 TFLOP/s).
    nnz = float(entries) if entries is not None else 0.0
    t_alu = 4.0 * K * nnz / 74.4e12
    return {"t_roof_ms": t_roof * 1e3, "t_step_ms": ms, "frac": t_roof * 1e3 / ms,
            "t_alu_sparse_ms": t_alu * 1e3,
            "bound": "tensor" if t_tc >= t_hbm else "hbm",
            "flops": flops, "bytes": b_alg, "P_tc_tflops": peaks["bf16_tflops"], "BW_hbm_gbs": peaks["hbm_gbs"],
            "U": U, "R": R, "bytes_fp32_vals_variant": b_build,
            "frac_fp32_vals_variant": max(t_tc, b_build / (peaks["hbm_gbs"] * 1e9)) * 1e3 / ms}


def measure_workload(tw, torch, dev, w, d, steps, warmup, flush, peaks, peak_kind, clocks=None, full=True):
    """Time one workload: the sparse step three ways, each kernel, both dense FFNs."""
    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    x, wg, wu, wd = (to_dev(d[k]) for k in ("x", "wg_t", "wu_t", "wd"))
    M, K, N, T, C = w.M, w.K, w.N, w.T, w.C
    tb = tw.TwellBuffers(M, K, N, T, C, device=dev)
    y = torch.empty(M, K, dtype=torch.float32, device=dev)
    words = torch.zeros(2, dtype=torch.int32).pin_memory()
    ctrl = tb.ctrl

    launches = [0]

    def step_async():
        tw.gate_pack(x, wg, tb)
        n1 = tw.last_launch_count()
        tw.ffn_fwd(x, wu, wd, tb, y)
        launches[0] += n1 + tw.last_launch_count()

    def step_read_status():
        # The whole step, then one D2H of the overflow count and the device flags
        # (checked on the host once the step's end event has completed).
        step_async()
        words.copy_(ctrl[:2], non_blocking=True)

    def check_words():
        n_over, flags = int(words[0]), int(words[1])
        if flags != 0 or n_over > tb.R_cap:
            raise RuntimeError(f"{w.name}: device flags 0x{flags:x}, n_over {n_over} (R_cap {tb.R_cap})")
        return n_over

    def step_sync_gate():
        tw.gate_pack(x, wg, tb, sync=True)      # syncs, reads n_over, checks capacity
        n1 = tw.last_launch_count()
        tw.ffn_fwd(x, wu, wd, tb, y)
        launches[0] += n1 + tw.last_launch_count()

    def timed(fn, after=None):
        out = []
        for i in range(steps):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            if after:
                after()
            out.append(a.elapsed_time(b))
        return sum(out) / len(out)

    # Correctness of the configuration before timing: capacity and device flags.
    step_read_status()
    torch.cuda.synchronize()
    n_over = check_words()
    st, _, _ = tw.read_status(tb)
    if st != tw.OK:
        raise RuntimeError(f"{w.name}: sparse path status {st}")
    stats = workload_stats(tb, w, T, C)
    U = unique_active_units(tb, C, T)

    for _ in range(warmup):
        step_read_status()
    torch.cuda.synchronize()
    launches[0] = 0
    if clocks is not None:
        with clocks:
            ms = timed(step_read_status, check_words)
    else:
        ms = timed(step_read_status, check_words)
    n_launches = launches[0]
    ms_async = timed(step_async)

    def timed_warm(fn):
        # No flush between steps: whatever of the weights L2 keeps stays (secondary number).
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) / steps

    ms_warm = timed_warm(step_async)
    ms_sync = timed(step_sync_gate)

    # Per-kernel durations: the same steps again with an event pair around
    # every kernel (events between kernels stop a launch from overlapping the
    # previous kernel's tail, so these steps are not the ones timed above).
    traces = []
    for i in range(steps):
        flush.fill_(i & 0xFF)
        tr = tw.KernelTrace(capacity=16)
        with tr:
            step_async()
        traces.append(tr)
    torch.cuda.synchronize()
    per_kernel = {}
    for tr in traces:
        for name, t in tr.times_ms():
            per_kernel.setdefault(name, []).append(t)
    kern_ms = {k: sum(v) / len(v) for k, v in per_kernel.items()}

    # The in-build dense tcgen05 FFN on the same inputs (same flush discipline):
    # h as bf16 hi + lo (held to the same accuracy rule as the sparse path), and
    # the plain bf16-h variant as a second, labelled number.
    h = torch.empty(M, 2 * N, dtype=torch.bfloat16, device=dev)
    yd = torch.empty(M, K, dtype=torch.float32, device=dev)
    for _ in range(warmup):
        tw.dense_ffn(x, wg, wu, wd, h, yd)
    dense_ms = timed(lambda: tw.dense_ffn(x, wg, wu, wd, h, yd))
    h1 = h.view(-1)[:M * N].view(M, N)
    for _ in range(warmup):
        tw.dense_ffn(x, wg, wu, wd, h1, yd, bf16_h=True)
    dense_bf16h_ms = timed(lambda: tw.dense_ffn(x, wg, wu, wd, h1, yd, bf16_h=True))
    del h, h1, yd

    # Sanity only: the same dense FFN with torch bf16 matmuls (cuBLAS) and
    # elementwise kernels, h rounded to bf16.
    def cublas_ffn():
        return ((x @ wu.t()) * torch.relu(x @ wg.t())) @ wd
    for _ in range(2):
        cublas_ffn()
    cublas_ms = timed(cublas_ffn)

    NT = N // T
    flops_gate = 2.0 * M * K * N
    entries = stats["twell_entries"]
    bytes_updown = (2.0 * M * K                      # x rows
                    + 2.0 * M * NT                   # counts
                    + 5.0 * entries                  # idx + fp32 value per listed entry
                    + 4.0 * K * U                    # unique W_u^T and W_d rows
                    + 4.0 * M * K)                   # y (fp32)
    kernels = {}
    for name, t in kern_ms.items():
        if name == "gate_twell_gemm":
            ach = flops_gate / (t * 1e-3) / 1e12
            kernels[name] = {"ms": t, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                             "algorithmic": flops_gate}
        elif name == "twell_updown":
            ach = bytes_updown / (t * 1e-3) / 1e9
            kernels[name] = {"ms": t, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": ach / peaks["hbm_gbs"], "algorithmic": bytes_updown,
                             "l2_gather_gbs": 4.0 * K * entries / (t * 1e-3) / 1e9}
        elif name in ("overflow_up_gemm", "overflow_down_gemm"):
            # dense-equivalent work of the slotted rows: one K x N product each
            # (the down GEMM runs it twice, over the hi and lo halves of h)
            f = 2.0 * n_over * K * N * (2 if name == "overflow_down_gemm" else 1)
            kernels[name] = {"ms": t, "bound": "tensor", "achieved": f / (t * 1e-3) / 1e12, "unit": "TFLOP/s",
                             "peak": peaks["bf16_tflops"], "frac": f / (t * 1e-3) / 1e12 / peaks["bf16_tflops"],
                             "algorithmic": f}
        else:
            kernels[name] = {"ms": t}
    dominant = max(kern_ms.items(), key=lambda kv: kv[1])[0]
    dom = kernels[dominant]
    roofline = {"kernel": dominant, "bound": dom.get("bound"), "achieved": dom.get("achieved"),
                "peak": dom.get("peak"), "unit": dom.get("unit"), "frac": dom.get("frac"),
                "traffic": profiled_traffic(dominant, w.name), "peak_source": peak_kind + " (burst)"}
    out = {
        "workload": w.name, "M": M, "K": K, "N": N, "T": T, "C": C, "R_cap": tb.R_cap,
        "ms_per_step": ms, "value": M / (ms * 1e-3),
        "ms_per_step_async": ms_async, "ms_per_step_sync_gate": ms_sync,
        "ms_per_step_warm_l2": ms_warm,
        "dense_cublas_sanity": {"ms_per_step": cublas_ms,
                                "variant": "torch bf16 matmuls (cuBLAS) + elementwise, h in bf16; sanity only"},
        "sparsity": stats, "unique_units_gathered": U, "n_over": n_over,
        "roofline": roofline,
        "path_roofline": path_roofline(M, K, N, T, C, U, n_over, peaks, ms, entries=stats["twell_entries"]),
        "kernels": kernels,
        "dense": {"ms_per_step": dense_ms, "value": M / (dense_ms * 1e-3), "unit": UNIT,
                  "variant": "dense_ffn_fwd: h as bf16 hi + lo, held to the same y rule as the sparse path"},
        "dense_bf16h": {"ms_per_step": dense_bf16h_ms, "value": M / (dense_bf16h_ms * 1e-3), "unit": UNIT,
                        "variant": "dense_ffn_fwd_bf16h: h rounded to one bf16 (not held to the y rule)"},
        "speedup_vs_dense": dense_ms / ms, "speedup_vs_dense_bf16h": dense_bf16h_ms / ms,
        "gpu_launches": n_launches,
    }
    out["_tensors"] = (x, wg, wu, wd, tb, y)
    return out


def measure_small_batch(tw, torch, dev, w, d, peaks, reps=25):
    """Per-step time of the small-batch paths: twell_ffn_fused (one persistent
    kernel after the reset), the two-call path (gate_pack + ffn_fwd) and both
    dense FFNs, each replayed from a CUDA graph of SMALL_BATCH_COPIES steps,
    step i on weight copy i (their total exceeds L2)."""
    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    M, K, N, T, C = w.M, w.K, w.N, w.T, w.C
    x = to_dev(d["x"])
    base = [to_dev(d[k]) for k in ("wg_t", "wu_t", "wd")]
    sets = [base] + [[t.clone() for t in base] for _ in range(SMALL_BATCH_COPIES - 1)]
    bufs = [tw.TwellBuffers(M, K, N, T, C, device=dev) for _ in range(SMALL_BATCH_COPIES)]
    ys = [torch.empty(M, K, dtype=torch.float32, device=dev) for _ in range(SMALL_BATCH_COPIES)]
    h = torch.empty(M, 2 * N, dtype=torch.bfloat16, device=dev)
    h1 = h.view(-1)[:M * N].view(M, N)

    def fused(i):
        tw.ffn_fused(x, *sets[i], bufs[i], ys[i])

    def two_call(i):
        tw.gate_pack(x, sets[i][0], bufs[i])
        tw.ffn_fwd(x, sets[i][1], sets[i][2], bufs[i], ys[i])

    def dense(i):
        tw.dense_ffn(x, *sets[i], h, ys[i])

    def dense1(i):
        tw.dense_ffn(x, *sets[i], h1, ys[i], bf16_h=True)

    out = {"workload": w.name, "M": M, "K": K, "N": N, "T": T, "C": C,
           "timing": f"CUDA graph of {SMALL_BATCH_COPIES} steps on {SMALL_BATCH_COPIES} weight copies "
                     f"({SMALL_BATCH_COPIES * 6 * K * N / 1e6:.0f} MB, more than L2), {reps} replays"}
    for name, fn in (("fused", fused), ("two_call", two_call), ("dense", dense), ("dense_bf16h", dense1)):
        for i in range(SMALL_BATCH_COPIES):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(SMALL_BATCH_COPIES):
                fn(i)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        b.synchronize()
        out[name] = {"ms_per_step": a.elapsed_time(b) / (reps * SMALL_BATCH_COPIES)}
        del g
    st, n_over, flags = tw.read_status(bufs[0])
    if st != tw.OK:
        raise RuntimeError(f"{w.name}: small-batch status {st} flags {flags}")
    U = unique_active_units(bufs[0], C, T)
    ms = out["fused"]["ms_per_step"]
    out["value"] = M / (ms * 1e-3)
    out["unit"] = UNIT
    out["n_over"] = n_over
    out["unique_units_gathered"] = U
    out["path_roofline"] = path_roofline(M, K, N, T, C, U, n_over, peaks, ms)
    out["speedup_vs_dense"] = out["dense"]["ms_per_step"] / ms
    out["speedup_vs_dense_bf16h"] = out["dense_bf16h"]["ms_per_step"] / ms
    return out


def measure_backward(tw, torch, dev, w, d, steps, warmup, flush, peaks):
    """twell_ffn_bwd after a synchronous gate pass: whole-call time (events,
    L2 flushed before each call), per-kernel times, and a dense backward of
    the same FFN with torch bf16 matmuls (cuBLAS) for context."""
    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    x, wg, wu, wd = (to_dev(d[k]) for k in ("x", "wg_t", "wu_t", "wd"))
    M, K, N, T, C = w.M, w.K, w.N, w.T, w.C
    tb = tw.TwellBuffers(M, K, N, T, C, device=dev)
    n_over = tw.gate_pack(x, wg, tb, sync=True)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    dy = torch.randn(M, K, device=dev, generator=g)
    need = tw.lib().twell_bwd_scratch_bytes(M, K, N, T, C, tb.R_cap)
    scratch = torch.empty(need, dtype=torch.uint8, device=dev)

    def bwd():
        return tw.ffn_bwd(x, wg, wu, wd, tb, dy, scratch)

    def dense_bwd():
        z = x @ wg.t()
        u = x @ wu.t()
        gg = torch.relu(z)
        dyb = dy.to(torch.bfloat16)
        dh = dyb @ wd.t()
        du = dh * gg
        dz = dh * u * (z > 0)
        return du @ wu + dz @ wg, dz.t() @ x, du.t() @ x, (u * gg).t() @ dyb

    def timed(fn, n):
        out = []
        for i in range(n):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            out.append(a.elapsed_time(b))
        return sum(out) / len(out)

    for _ in range(warmup):
        bwd()
    ms = timed(bwd, steps)
    per = {}
    for i in range(min(steps, 5)):
        flush.fill_(i & 0xFF)
        tr = tw.KernelTrace(capacity=16)
        with tr:
            bwd()
        torch.cuda.synchronize()
        for name, t in tr.times_ms():
            per.setdefault(name, []).append(t)
    for _ in range(2):
        dense_bwd()
    dense_ms = timed(dense_bwd, min(steps, 5))
    st, _, _ = tw.read_status(tb)
    stats = workload_stats(tb, w, T, C)
    return {"workload": w.name, "M": M, "K": K, "N": N, "ms": ms, "tokens_per_s": M / (ms * 1e-3),
            "n_over": n_over, "twell_entries": stats["twell_entries"], "status": st,
            "kernels_ms": {k: sum(v) / len(v) for k, v in per.items()},
            # which route the library chose for the slotted rows (seen in the trace)
            "slotted_rows_route": "dense-slot GEMMs" if any(k.startswith("bwd_slot_") for k in per)
                                  else "gather passes",
            "torch_dense_backward_ms": dense_ms,
            "torch_dense_backward": "bf16 torch matmuls (cuBLAS) and elementwise ops, recomputing z and u; "
                                    "context only, not held to the y rule",
            "speedup_vs_torch_dense": dense_ms / ms}


def run_ncu_case(args):
    """The sparse path only, --warmup + 1 times, on one GPU: the launches an
    ncu capture selects from (no flush buffer, no dense FFN, no timing)."""
    import torch

    from activation_sparse_gated_tma_b200 import twell as tw

    w = wl.WORKLOADS[args.workload]
    d = wl.generate(w)
    dev = {k: torch.from_numpy(d[k].view(np.int16)).view(torch.bfloat16).cuda() for k in ("x", "wg_t", "wu_t", "wd")}
    tb = tw.TwellBuffers(w.M, w.K, w.N, w.T, w.C)
    y = torch.empty(w.M, w.K, dtype=torch.float32, device="cuda")
    dy = torch.randn(w.M, w.K, device="cuda") if args.ncu_backward else None
    if args.ncu_backward:
        tw.gate_pack(dev["x"], dev["wg_t"], tb, sync=True)
    for _ in range(args.warmup + 1):
        if args.ncu_backward:
            tw.ffn_bwd(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], tb, dy)
        elif args.ncu_fused:
            tw.ffn_fused(dev["x"], dev["wg_t"], dev["wu_t"], dev["wd"], tb, y)
        else:
            tw.gate_pack(dev["x"], dev["wg_t"], tb)
            tw.ffn_fwd(dev["x"], dev["wu_t"], dev["wd"], tb, y)
    st, n_over, flags = tw.read_status(tb)
    if st != tw.OK:
        raise RuntimeError(f"status {st} (n_over {n_over}, flags {flags})")
    print(json.dumps({"ncu_case": w.name, "passes": args.warmup + 1, "n_over": n_over,
                      "call": "twell_ffn_bwd" if args.ncu_backward else
                      ("twell_ffn_fused" if args.ncu_fused else "twell_gate_pack + twell_ffn_fwd")}))


def run_sweep(args):
    """One JSON line per sweep workload, on one GPU, timed as the small-batch
    block (CUDA graph over rotating weight copies)."""
    import torch

    from activation_sparse_gated_tma_b200 import twell as tw

    peaks, _ = load_peaks()
    dev = torch.device("cuda", 0)
    for name in sorted(n for n in wl.WORKLOADS if n.startswith("sweep_")):
        w = wl.WORKLOADS[name]
        r = measure_small_batch(tw, torch, dev, w, wl.generate(w), peaks)
        print(json.dumps({"sweep": name, "M": w.M, "fused_ms": r["fused"]["ms_per_step"],
                          "two_call_ms": r["two_call"]["ms_per_step"], "dense_ms": r["dense"]["ms_per_step"],
                          "dense_bf16h_ms": r["dense_bf16h"]["ms_per_step"], "speedup_vs_dense": r["speedup_vs_dense"],
                          "path_roofline_frac": r["path_roofline"]["frac"], "n_over": r["n_over"]}), flush=True)
        torch.cuda.empty_cache()


def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from activation_sparse_gated_tma_b200 import twell as tw

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, peak_kind = load_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    w = wl.WORKLOADS[args.workload]
    d = wl.generate(w)
    clk = ClockSampler(local_rank)
    head = measure_workload(tw, torch, dev, w, d, args.steps, args.warmup, flush, peaks, peak_kind, clocks=clk)
    x, wg, wu, wd, tb, y = head.pop("_tensors")

    # End to end through the public API with host buffers: pinned x in, y out,
    # plus the overflow count and device flags (twell_read_status).
    x_host = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty(w.M, w.K, dtype=torch.float32).pin_memory()
    x_e2e = torch.empty_like(x)
    words = torch.zeros(2, dtype=torch.int32).pin_memory()

    def e2e_step():
        x_e2e.copy_(x_host, non_blocking=True)
        tw.gate_pack(x_e2e, wg, tb)
        tw.ffn_fwd(x_e2e, wu, wd, tb, y)
        y_host.copy_(y, non_blocking=True)
        words.copy_(tb.ctrl[:2], non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    e2e_ms = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        e2e_step()
        b.record()
        b.synchronize()
        if int(words[1]) != 0 or int(words[0]) > tb.R_cap:
            raise RuntimeError(f"end-to-end step: device flags {int(words[1])}, n_over {int(words[0])}")
        e2e_ms.append(a.elapsed_time(b))
    e2e_ms = sum(e2e_ms) / len(e2e_ms)
    del x, wg, wu, wd, tb, y, x_e2e

    # The other full-size workloads, measured the same way (same steps).
    others = {}
    if not args.no_extra:
        for name in EXTRA_WORKLOADS:
            if name == w.name:
                continue
            wo = wl.WORKLOADS[name]
            r = measure_workload(tw, torch, dev, wo, wl.generate(wo), args.steps, args.warmup, flush, peaks,
                                 peak_kind)
            r.pop("_tensors")
            others[name] = r
            torch.cuda.empty_cache()

    small = {}
    if not args.no_extra:
        for name in SMALL_BATCH_WORKLOADS:
            ws = wl.WORKLOADS[name]
            small[name] = measure_small_batch(tw, torch, dev, ws, wl.generate(ws), peaks)
            torch.cuda.empty_cache()

    backward = {}
    if not args.no_extra:
        for name in BACKWARD_WORKLOADS:
            wb = wl.WORKLOADS[name]
            backward[name] = measure_backward(tw, torch, dev, wb, wl.generate(wb), args.steps, args.warmup, flush,
                                              peaks)
            torch.cuda.empty_cache()

    # One collective on every rank: the job's time is the slowest rank's.
    ms, e2e_ms = max_over_ranks([head["ms_per_step"], e2e_ms], world, dev)
    if rank != 0:
        return

    cpu = None
    if not args.no_cpu_baseline:
        rate, rows, sec, cores = cpu_oracle_rate(d, w, rows_target_s=12.0)
        drate, drows, dsec = cpu_dense_oracle_rate(d, w)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
               "sample": f"{rows} seeded rows of {w.M} ({sec:.1f} s): fp64 gate, TwELL pack, sparse y",
               "dense_oracle": {"value": drate, "unit": UNIT,
                                "sample": f"{drows} seeded rows ({dsec:.1f} s): fp64 dense FFN, every hidden unit"}}

    value = job_throughput(world, w.M, ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "T": w.T, "C": w.C, "R_cap": head["R_cap"],
                   "global_batch": world * w.M, "parallelism": f"replicas{world}",
                   "l2": "flushed: 256 MiB write before each timed step (outside the timed events)",
                   "mode": "step = twell_gate_pack + twell_ffn_fwd + one D2H of the overflow count and device "
                           "flags, checked on the host after the step (capacity retry on overflow)"},
        "ms_per_step_async": head["ms_per_step_async"], "ms_per_step_sync_gate": head["ms_per_step_sync_gate"],
        "sparsity": head["sparsity"], "unique_units_gathered": head["unique_units_gathered"],
        "n_over": head["n_over"],
        "roofline": head["roofline"],
        "path_roofline": path_roofline(w.M, w.K, w.N, w.T, w.C, head["unique_units_gathered"], head["n_over"],
                                       peaks, ms, entries=head["sparsity"]["twell_entries"]),
        "ms_per_step_warm_l2": head["ms_per_step_warm_l2"],
        "dense_cublas_sanity": head["dense_cublas_sanity"],
        "kernels": head["kernels"],
        "dense": head["dense"], "dense_bf16h": head["dense_bf16h"],
        "speedup_vs_dense": head["dense"]["ms_per_step"] / ms,
        "speedup_vs_dense_bf16h": head["dense_bf16h"]["ms_per_step"] / ms,
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(world, w.M, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": 2 * w.M * w.K,
                "d2h_bytes_per_step": 4 * w.M * w.K + 8, "ms_per_step": e2e_ms},
        "gpu_launches": head["gpu_launches"],
        "clocks": clk.summary(),
        "other_workloads": others,
        "small_batch": small,
        "backward": backward,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=wl.BENCH_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="time only --workload")
    ap.add_argument("--ncu-case", action="store_true",
                    help="no timing: --warmup + 1 passes of the sparse path on --workload (for ncu captures)")
    ap.add_argument("--ncu-fused", action="store_true", help="with --ncu-case: the passes call twell_ffn_fused")
    ap.add_argument("--ncu-backward", action="store_true",
                    help="with --ncu-case: one synchronous gate pass, then the passes call twell_ffn_bwd")
    ap.add_argument("--sweep", action="store_true",
                    help="print one JSON line per sweep workload (M 16..4096, 90/99/99.9%% sparsity), timed "
                         "like the small-batch block, instead of the bench line")
    args = ap.parse_args()
    if args.warmup < 3 and not args.ncu_case:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.ncu_case:
        run_ncu_case(args)
        return
    if args.sweep:
        run_sweep(args)
        return

    import datetime

    import torch.distributed as dist
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
