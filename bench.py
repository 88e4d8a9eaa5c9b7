"""Benchmark of the FP8 dynamic-quantisation linear path on B200.

One step = one pass of the whole hot path over one batch of seeded synthetic
input, the prefill-shaped linear workload: bf16 activations X[4096,7168]
(N(0,1), 72 columns x50) resident in HBM ->
    per-tensor quantisation (amax pass + apply pass)      -> codes + 1 scale
    per-1x128-group quantisation                          -> codes + [4096,56] scales
    block-scaled FP8 GEMM against E4M3 weights B[N,7168] with 128x128 block
    scales, for N = 7168, 18432, 24576                    -> bf16 Y[4096,N]
Weight quantisation is an offline step and is not timed.  Inputs per step
(X and the three weights, 419 MB) exceed the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --op gemm --m 4096 --n 7168 --k 7168 [--reps R] [--modes cold,graph]

Prints ONE JSON line (rank 0).  `value` is the whole-job GEMM throughput of
the step (2*M*sum(N)*K flops over the device-timed step, all ranks);
per-kernel times inside the step are in `kernels`, and `workloads` holds
every other workload's kernels timed on their own (CUDA-graph replay, as the
pages timed their amax kernel, and with L2 flushed for the large ones).
`--impl reference` times the CPU oracle on the host cores on a bounded
sample of the same workload.  Multi-GPU (torchrun): every rank runs its own
batch (weak scaling, no collective on the data path); time = max over ranks.
With more than one rank the row-sharded per-tensor quantisation (local amax,
one 4-byte MAX all-reduce, local apply) is also timed.

`--op` times one operation at one shape and prints one JSON line per timing
mode (the commands behind the ncu summaries in profiles/ use it).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_dynamic_quantization_b200 import inputs  # noqa: E402

METRIC = "quant GB/s and FP8 block GEMM TFLOPS at 1 B200; % of HBM / FP8-tensor roofline"
M, K = 4096, 7168
NS = (7168, 18432, 24576)
WORKLOAD = ("prefill linear step: bf16 X[4096,7168] -> per-tensor quant (amax+apply) -> "
            "group-128 quant -> block-scaled FP8 GEMM vs B[N,7168] for N in {7168,18432,24576}")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0            # nominal dense ratio 4.5 / 2.25 PFLOP/s
L2_BYTES = 126 * 2 ** 20
# The pages' B200 per-tensor amax kernel (fixed-size grid replaced by an
# input-sized one), us per call under CUDA graph, K = 2048 ("Size the
# per-tensor FP8 dynamic-quant amax grid to the input", Test Coverage).
PAGE_AMAX_US = {1: 4.1, 64: 4.1, 256: 6.1, 1024: 6.1, 65536: 43.0}


def gemm_flops(m=M, ns=NS, k=K):
    return sum(2.0 * m * n * k for n in ns)


# Algorithmic bytes per launch (what the method must move at least once).
def bytes_per_tensor(m=M, k=K, unique=False):
    """amax read 2 B + apply read 2 B + code write 1 B per element; with
    unique=True the second read is not counted (3 B/element: the tensor
    fits in L2, so the apply pass can re-read it from there)."""
    return (3.0 if unique else 5.0) * m * k + 4


def bytes_amax(m, k):
    return 2.0 * m * k


def bytes_group128(m=M, k=K):         # read 2B + write 1B per element + one fp32 per 128
    return 3.0 * m * k + 4.0 * m * (k // 128)


def bytes_gemm(m, n, k=K):
    g = k // 128
    return m * k + n * k + 4.0 * m * g + 4.0 * ((n + 127) // 128) * g + 2.0 * m * n


GEMM_SOURCES = ("gemm_kernels.cuh", "ptx_sm100.cuh", "launch_table.inc")
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "block_gemm_prefill_4096xNx7168.md")


def code_digest(texts) -> str:
    """sha256 (first 16 hex digits) of C/C++ sources with comments removed
    and whitespace collapsed: edits to comments or layout keep the digest,
    any change to the code changes it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for t in texts:
        t = re.sub(r"/\*.*?\*/", " ", t, flags=re.S)        # block comments
        t = re.sub(r"//[^\n]*", " ", t)                      # line comments
        h.update(" ".join(t.split()).encode())
    return h.hexdigest()[:16]


def gemm_traffic():
    """DRAM bytes per GEMM launch (mean over the step's three launches) from
    the committed ncu summary -- only while the GEMM code still has the
    digest recorded there; None otherwise."""
    csrc = os.path.join(ROOT, "fp8_dynamic_quantization_b200", "csrc")
    try:
        texts = []
        for f in GEMM_SOURCES:
            with open(os.path.join(csrc, f)) as fh:
                texts.append(fh.read())
        rec = {}
        with open(TRAFFIC_RECORD) as fh:
            for line in fh:
                if ":" in line and line.split(":", 1)[0].strip() in (
                        "gemm_code_digest", "dram_bytes_per_launch_mean"):
                    k, v = line.split(":", 1)
                    rec[k.strip()] = v.split()[0]
    except OSError:
        return None
    if rec.get("gemm_code_digest") != code_digest(texts):
        return None
    return float(rec["dram_bytes_per_launch_mean"])


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def parse_clock_rows(text, t0=None, t1=None):
    """Summary of nvidia-smi CSV rows (timestamp first, then ClockSampler's
    fields): median SM clock, max clock, active throttle reasons.  Only rows
    stamped inside [t0, t1] (host wall-clock seconds, the timed region) count
    when t0/t1 are given and any row falls inside; otherwise all rows count."""
    import datetime
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    rows = []
    for line in text.strip().splitlines():
        r = [c.strip() for c in line.split(",")]
        if len(r) < 10:
            continue
        try:
            ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            ts = None
        rows.append((ts, r[1:]))
    if not rows:
        return None
    inside = [r for ts, r in rows if t0 is not None and ts is not None and t0 <= ts <= t1]
    use = inside if inside else [r for _, r in rows]
    sm = [float(r[1]) for r in use if r[1].replace(".", "").isdigit()]
    mx = [float(r[2]) for r in use if r[2].replace(".", "").isdigit()]
    reasons = sorted({names[i] for r in use for i in range(4) if r[5 + i] == "Active"})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons, "samples": len(use), "in_timed_region": bool(inside)}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every `interval_ms`; the
    summary keeps the samples stamped inside the timed region."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, interval_ms: int = 10):
        self.index = index
        self.interval_ms = interval_ms
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)                      # first samples before the timed region

    def mark(self, begin: bool):
        """Host wall-clock bounds of the timed region."""
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return parse_clock_rows(out, self.t0, self.t1)


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ---------------------------------------------------------------- timers
class Timer:
    """Device time of one call, CUDA events on the launching stream.

    cold : an L2 flush (reading a 256 MB buffer, which leaves only clean
           lines in L2) and a GPU sleep before every call, outside the timed
           interval (the sleep hides the host's launch overhead); median of
           `reps` calls.
    graph: `reps` calls captured in one CUDA graph and replayed; time / reps
           (how the pages timed their amax kernel; inputs that fit in L2 stay
           L2-warm).
    stream: like graph, but the calls cycle over several copies of the
           inputs whose total exceeds L2, so every call reads its input from
           HBM while its launch overlaps the previous call as in a step (no
           event or host gap between calls)."""

    def __init__(self, dev):
        self.dev = dev
        self.flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def cold(self, fn, reps):
        fn()                          # untimed: first-call set-up (workspace, tensor maps)
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            self.flush_buf.max()
            torch.cuda._sleep(200_000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    def graph(self, fn, reps):
        return self.stream([fn], reps)

    def stream(self, fns, reps, replays=1):
        """Graph of `reps` calls cycling over `fns`; time per call (median
        of `replays` replays)."""
        for fn in fns:
            fn()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for fn in fns:
                fn()                  # populate per-stream workspace caches
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(reps):
                fns[i % len(fns)]()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(replays):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / reps)
        del g
        return statistics.median(ts)


# ---------------------------------------------------------------- operations
def _dev_codes(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev).view(torch.float8_e4m3fn)


def _dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def _out(m, n, dev):
    """bf16 [m, n] output with a 16-byte row pitch."""
    return torch.empty(m, (n + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :n]


def input_copies(nbytes):
    """Copies of an input that together exceed L2 twice over (at least 2,
    at most 8), for the rotating `stream` timing."""
    return int(min(8, max(2, -(-2 * L2_BYTES // max(1, int(nbytes))))))


def make_op(op, m, n, k, dev, copies=1):
    """(callables, algorithmic bytes, flops or None, extra record fields) for
    one operation at one shape, on seeded synthetic inputs of its workload.
    The quantisation ops get `copies` callables, each on its own copy of the
    input (the others get one)."""
    import fp8_dynamic_quantization_b200 as fq

    def xs(x):
        x = x.to(dev)
        return [x] + [x.clone() for _ in range(copies - 1)]
    if op == "per_tensor":
        return [(lambda x=x: fq.act_quant_per_tensor(x)) for x in xs(inputs.activations_per_tensor(m, k=k))], \
            bytes_per_tensor(m, k), None, {
                "GB/s_basis": "5 B/element (amax read + apply read + code write)",
                "unique_bytes": bytes_per_tensor(m, k, unique=True)}
    if op == "amax":
        return [(lambda x=x: fq.act_amax(x)) for x in xs(inputs.activations_per_tensor(m, k=k))], \
            bytes_amax(m, k), None, {}
    if op == "group128":
        return [(lambda x=x: fq.act_quant_group128(x)) for x in xs(inputs.activations_group(m, k=k))], \
            bytes_group128(m, k), None, {}
    if op == "group128_ue8m0":
        return [(lambda x=x: fq.act_quant_group128_ue8m0(x)) for x in xs(inputs.activations_group(m, k=k))], \
            3.0 * m * k + m * (k // 128), None, {}
    if op == "per_channel":
        return [(lambda x=x: fq.act_quant_per_channel(x)) for x in xs(inputs.activations_per_tensor(m, k=k))], \
            3.0 * m * k + 4.0 * m, None, {}
    flops = 2.0 * m * n * k
    if op == "gemm":
        qa, sa, qb, sb = inputs.gemm_operands(m, n, k)
        tqa, tqb, tsa, tsb = _dev_codes(qa, dev), _dev_codes(qb, dev), _dev(sa, dev), _dev(sb, dev)
        y = _out(m, n, dev)
        return [lambda: fq.block_gemm(tqa, tsa, tqb, tsb, out=y)], bytes_gemm(m, n, k), flops, {}
    if op in ("gemm_pt", "gemm_pc", "gemm_ue8m0"):
        qa, _, qb, _ = inputs.gemm_operands(m, n, k)
        tqa, tqb = _dev_codes(qa, dev), _dev_codes(qb, dev)
        y = _out(m, n, dev)
        g = inputs.rng(m + n)
        if op == "gemm_pt":
            sa, sb = torch.tensor([0.01], device=dev), torch.tensor([0.02], device=dev)
            return [lambda: fq.gemm_per_tensor(tqa, sa, tqb, sb, out=y)], \
                m * k + n * k + 8.0 + 2.0 * m * n, flops, {}
        if op == "gemm_pc":
            sa = _dev(g.uniform(1e-3, 1e-1, m).astype(np.float32), dev)
            sb = _dev(g.uniform(1e-3, 1e-1, n).astype(np.float32), dev)
            return [lambda: fq.gemm_per_channel(tqa, sa, tqb, sb, out=y)], \
                m * k + n * k + 4.0 * (m + n) + 2.0 * m * n, flops, {}
        sa = _dev(g.integers(115, 135, (m, k // 128)).astype(np.uint8), dev)
        sb = _dev(g.integers(115, 135, ((n + 127) // 128, k // 128)).astype(np.uint8), dev)
        return [lambda: fq.block_gemm_ue8m0(tqa, sa, tqb, sb, out=y)], \
            m * k + n * k + m * k / 128 + ((n + 127) // 128) * k / 128 + 2.0 * m * n, flops, {}
    if op == "linear":
        # the one-call group-128 linear: quantisation kernel, then the GEMM
        # launched as its programmatic dependent
        x = inputs.activations_group(m, k=k).to(dev)
        qb, sb = inputs.weight_operands(n, k)
        tqb, tsb = _dev_codes(qb, dev), _dev(sb, dev)
        y = _out(m, n, dev)
        return [lambda: fq.linear_fused(x, tqb, tsb, out=y)], \
            2.0 * m * k + n * k + 4.0 * ((n + 127) // 128) * (k // 128) + 2.0 * m * n, flops, {}
    raise ValueError(op)


QUANT_OPS = ("per_tensor", "amax", "group128", "group128_ue8m0", "per_channel")


def time_op(timer, op, m, n, k, dev, modes, reps, hbm, fp8_peak):
    copies = input_copies(2.0 * m * k) if (op in QUANT_OPS and "stream" in modes) else 1
    fns, nbytes, flops, extra = make_op(op, m, n, k, dev, copies)
    out = []
    for mode in modes:
        if mode == "stream" and op not in QUANT_OPS:
            continue
        us = timer.stream(fns, reps, replays=3) if mode == "stream" else getattr(timer, mode)(fns[0], reps)
        rec = {"op": op, "M": m, "N": n, "K": k, "mode": mode, "us": us,
               "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm}
        if "unique_bytes" in extra:
            rec["GB/s_unique"] = extra["unique_bytes"] / us / 1e3
            rec["frac_hbm_unique"] = rec["GB/s_unique"] / hbm
        if flops:
            rec["TFLOP/s"] = flops / us / 1e6
            rec["frac_fp8"] = flops / us / 1e6 / fp8_peak
        if mode == "stream":
            rec["input_copies"] = copies
        out.append(rec)
    del fns
    return out


def fp8_peak_cublaslt(dev, n=8192):
    """cuBLASLt's per-tensor-scaled FP8 GEMM (torch._scaled_mm, E4M3 in,
    bf16 out) at n^3 on random data: best of 10 calls, in TFLOP/s.  The
    measured denominator for FP8 contractions on this GPU."""
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    one = torch.tensor(1.0, device=dev)

    def f():
        return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(5):
        f()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        f()
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def workload_table(dev, hbm, fp8_peak, reps=20):
    """Every workload's kernels timed on their own (graph replay; L2-flushed
    'cold' timing too where the data exceed L2)."""
    timer = Timer(dev)
    rows = []

    def add(op, m, n, k, big):
        modes = ["graph", "cold", "stream"] if big else ["graph"]
        rows.extend(time_op(timer, op, m, n, k, dev, modes, reps, hbm, fp8_peak))
    # workload 1: the tiny linear layer
    add("per_tensor", 64, 0, 2048, False)
    add("group128", 64, 0, 2048, False)
    add("gemm", 64, 2048, 2048, False)
    # workload 2: per-tensor sweep, whole path and the amax alone (the pages' kernel)
    for m in (1, 64, 256, 1024, 65536):
        big = m * 2048 * 2 > L2_BYTES // 2
        add("per_tensor", m, 0, 2048, big)
        before = len(rows)
        add("amax", m, 0, 2048, big)
        for r in rows[before:]:
            r["page_amax_us"] = PAGE_AMAX_US[m]
    # workload 3: group-128 sweep
    for m in (1, 32, 4096, 16384):
        add("group128", m, 0, 7168, m >= 4096)
    # workload 4: decode GEMM
    for m in (1, 16, 64, 256):
        for n in (2048, 7168, 18432):
            add("gemm", m, n, 7168, n == 18432)
    # the other scale formats and the one-call linear, decode and prefill
    for op in ("gemm_pt", "gemm_ue8m0", "gemm_pc"):
        add(op, 16, 18432, 7168, False)
        add(op, 4096, 18432, 7168, False)
    add("linear", 16, 18432, 7168, False)
    add("linear", 4096, 18432, 7168, False)
    for op in ("group128_ue8m0", "per_channel"):
        add(op, 16384, 0, 7168, True)
    del timer
    return rows


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(rows: int, x_bits: np.ndarray, weights):
    """The oracle over a row sample of the step: per-tensor and group-128
    quantisation of `rows` rows and the GEMM of those rows for every N."""
    import oracle
    xs = np.ascontiguousarray(x_bits[:rows])
    oracle.quant_per_tensor(xs)
    qa, sa = oracle.quant_group128(xs)
    for qb, sb in weights:
        oracle.block_gemm(qa, sa, qb, sb)
    return gemm_flops(rows)


def cpu_baseline(x_bits, weights, budget_s=10.0):
    import oracle
    threads = oracle.set_threads(0)
    t0 = time.perf_counter()
    oracle_sample(1, x_bits, weights)
    one = time.perf_counter() - t0
    rows = int(max(1, min(M, budget_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    flops = oracle_sample(rows, x_bits, weights)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows} of {M} rows of the step (per-tensor + group-128 quant of those rows, "
                      f"float64 block GEMM of those rows for N in {list(NS)}); {dt:.1f} s"}


def reference_arm(args, rank, world):
    """`--impl reference`: the CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return
    import oracle
    threads = oracle.set_threads(0)
    x_bits = inputs.bf16_bits(inputs.activations_prefill())
    weights = [inputs.weight_operands(n) for n in NS]
    t0 = time.perf_counter()
    oracle_sample(1, x_bits, weights)
    one = time.perf_counter() - t0
    # each step: a row sample sized so warm-up + timed steps fit in ~3 minutes
    rows = int(max(1, min(M, 180.0 / max(one, 1e-3) / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        oracle_sample(rows, x_bits, weights)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(rows, x_bits, weights)
    dt = time.perf_counter() - t0
    value = gemm_flops(rows) * args.steps / dt / 1e12
    sample = f"{rows} of {M} rows per step (quantisation + float64 GEMM of those rows, all N)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": list(NS), "parallelism": "none"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------- GPU arm
def sharded_per_tensor(x, dist, steps, warmup, stream):
    """Row-sharded per-tensor quantisation across the ranks (each rank's X is
    its shard): local amax, one 4-byte MAX all-reduce over NCCL, local
    apply.  Device time per call, max over ranks."""
    import fp8_dynamic_quantization_b200 as fq
    for _ in range(warmup):
        fq.per_tensor_sharded(x)
    torch.cuda.synchronize()
    dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fq.per_tensor_sharded(x)
    b.record(stream)
    torch.cuda.synchronize()
    t = torch.tensor([a.elapsed_time(b) / steps], dtype=torch.float64, device=x.device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def our_arm(args, rank, world, local_rank):
    import fp8_dynamic_quantization_b200 as fq
    lib = fq.library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    x_cpu = inputs.activations_prefill(seed=5000 + rank)
    x = x_cpu.to(dev)
    weights_np = [inputs.weight_operands(n, seed=5100 + 1000 * rank) for n in NS]
    weights = [(torch.from_numpy(qb).to(dev).view(torch.float8_e4m3fn), torch.from_numpy(sb).to(dev))
               for qb, sb in weights_np]
    ys = [torch.empty(M, n, dtype=torch.bfloat16, device=dev) for n in NS]
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fq.act_quant_per_tensor(x)
        if ev is not None:
            ev[1].record(stream)
        qa, sa = fq.act_quant_group128(x)
        if ev is not None:
            ev[2].record(stream)
        for i, (qb, sb) in enumerate(weights):
            fq.block_gemm(qa, sa, qb, sb, out=ys[i])
            if ev is not None:
                ev[3 + i].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if fq.device_status() != 0:
        raise RuntimeError("device-side error during warm-up")

    nev = 3 + len(NS)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else
                          (f"GPU-{uuid}" if uuid else str(local_rank)))
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = lib.fp8q_launch_count()
    clocks.mark(True)
    start.record(stream)
    for s in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark(False)
    launches = lib.fp8q_launch_count() - launches0
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    ms = start.elapsed_time(end)
    if fq.device_status() != 0:
        raise RuntimeError("device-side error during the timed steps")

    # Per-kernel times: a second pass of the same steps with an event between
    # every two calls (the timed region above has none, so that each launch
    # can overlap the tail of the one before it).
    for s in range(args.steps):
        step(events[s])
    torch.cuda.synchronize(dev)

    # per-kernel averages (ms) from the in-stream events
    def avg(i, j):
        return sum(events[s][i].elapsed_time(events[s][j]) for s in range(args.steps)) / args.steps
    k_ms = {"per_tensor_quant": avg(0, 1), "group128_quant": avg(1, 2)}
    for i, n in enumerate(NS):
        k_ms[f"gemm_N{n}"] = avg(2 + i, 3 + i)
    # What an event pair costs by itself: the same bracketing around an
    # empty kernel.
    floor_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(50)]
    for a, b in floor_ev:
        a.record(stream)
        torch.cuda._sleep(0)
        b.record(stream)
    torch.cuda.synchronize(dev)
    event_floor_ms = statistics.median(a.elapsed_time(b) for a, b in floor_ev)
    # The quantisation kernels back to back as in the step (launches
    # overlapping, no events between them) on copies of X that together
    # exceed L2, so every call reads its X from HBM.
    timer = Timer(dev)
    x_copies = [x] + [x.clone() for _ in range(input_copies(x.numel() * 2) - 1)]
    pipe_ms = {
        "per_tensor_quant": timer.stream([(lambda t=t: fq.act_quant_per_tensor(t)) for t in x_copies],
                                         40, replays=5) * 1e-3,
        "group128_quant": timer.stream([(lambda t=t: fq.act_quant_group128(t)) for t in x_copies],
                                       40, replays=5) * 1e-3}
    del timer, x_copies

    if dist is not None:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    # ------------------------------------------------------------ e2e
    # Same step through the public API from pinned host memory: every step
    # copies its X to the device, runs the step and reads every Y back, all
    # inside the timed region.  The copies run on their own streams and the
    # device buffers alternate between two sets, so step i's output copies
    # overlap step i+1's kernels (PCIe is the bound: 411 MB of Y per step).
    x_host = x_cpu.pin_memory()
    y_host = [torch.empty(M, n, dtype=torch.bfloat16).pin_memory() for n in NS]
    x_devs = [torch.empty_like(x), torch.empty_like(x)]
    y_devs = [[torch.empty_like(y) for y in ys], [torch.empty_like(y) for y in ys]]
    copy_in = torch.cuda.Stream(device=dev)
    copy_out = torch.cuda.Stream(device=dev)
    x_free = [None, None]                        # set b's X no longer read
    y_free = [[None] * len(NS), [None] * len(NS)]  # set b's Y[j] copied out

    def mark(st):
        ev = torch.cuda.Event()
        ev.record(st)
        return ev

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(copy_in):
            if x_free[b] is not None:
                copy_in.wait_event(x_free[b])
            x_devs[b].copy_(x_host, non_blocking=True)
            x_in = mark(copy_in)
        stream.wait_event(x_in)
        fq.act_quant_per_tensor(x_devs[b])
        qa, sa = fq.act_quant_group128(x_devs[b])
        x_free[b] = mark(stream)
        for j, (qb, sb) in enumerate(weights):
            if y_free[b][j] is not None:
                stream.wait_event(y_free[b][j])
            fq.block_gemm(qa, sa, qb, sb, out=y_devs[b][j])
            y_ready = mark(stream)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(y_ready)
                y_host[j].copy_(y_devs[b][j], non_blocking=True)
                y_free[b][j] = mark(copy_out)

    def e2e_join():
        stream.wait_event(mark(copy_out))

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(3):
        e2e_step(i)
    e2e_join()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e2e_join()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if dist is not None:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = x.numel() * 2
    d2h = sum(M * n * 2 for n in NS)
    del x_host, y_host, x_devs, y_devs

    # ------------------------------------------------------------ the one exchange (N > 1)
    sharded_ms = None
    if dist is not None:
        sharded_ms = sharded_per_tensor(x, dist, max(10, args.steps), args.warmup, stream)

    peaks, peak_src = load_peaks()
    result = None
    table = None
    fp8_meas = None
    if rank == 0 and not args.no_kernels and world == 1:
        del ys
        torch.cuda.empty_cache()
        fp8_meas = fp8_peak_cublaslt(dev)
        table = workload_table(dev, peaks["hbm_gbs"], peaks["bf16_tflops"] * FP8_OVER_BF16)
    if rank == 0:
        step_ms = ms / args.steps
        total_flops = gemm_flops() * world
        value = total_flops / (step_ms * 1e-3) / 1e12
        hbm = peaks["hbm_gbs"]
        t_pt = pipe_ms["per_tensor_quant"]
        t_g = pipe_ms["group128_quant"]
        kernels = {
            "timing": "GEMMs: in-stream events between the calls of a second pass over the same steps. "
                      "Quantisation kernels (ms): the kernel alone back to back as in the step, launches "
                      "overlapping, on copies of X that together exceed L2 (each call reads its X from "
                      "HBM); ms_with_events: the second pass's event pair around the call, which also "
                      "holds the event pair's own cost (event_floor_ms, measured around an empty kernel)",
            "event_floor_ms": event_floor_ms,
            "per_tensor_quant": {
                "ms": t_pt,
                "ms_with_events": k_ms["per_tensor_quant"],
                "GB/s": bytes_per_tensor() / (t_pt * 1e-3) / 1e9,
                "GB/s_unique": bytes_per_tensor(unique=True) / (t_pt * 1e-3) / 1e9,
                "basis": "GB/s at 5 B/element (amax read, apply read, code write); GB/s_unique at "
                         "3 B/element (X, 58.7 MB, fits in L2: the apply pass may re-read it there)"},
            "group128_quant": {"ms": t_g, "ms_with_events": k_ms["group128_quant"],
                               "GB/s": bytes_group128() / (t_g * 1e-3) / 1e9},
        }
        kernels["per_tensor_quant"]["frac_hbm"] = kernels["per_tensor_quant"]["GB/s"] / hbm
        kernels["per_tensor_quant"]["frac_hbm_unique"] = kernels["per_tensor_quant"]["GB/s_unique"] / hbm
        kernels["group128_quant"]["frac_hbm"] = kernels["group128_quant"]["GB/s"] / hbm
        timed_s = ms * 1e-3
        bf16_peak = peaks["bf16_tflops"] if timed_s < 5.0 else peaks["bf16_tflops_sustained"]
        fp8_peak = bf16_peak * FP8_OVER_BF16
        for n in NS:
            t = k_ms[f"gemm_N{n}"]
            kernels[f"gemm_N{n}"] = {"ms": t, "TFLOP/s": 2.0 * M * n * K / (t * 1e-3) / 1e12,
                                     "GB/s": bytes_gemm(M, n) / (t * 1e-3) / 1e9}
            kernels[f"gemm_N{n}"]["frac_fp8"] = kernels[f"gemm_N{n}"]["TFLOP/s"] / fp8_peak
            if fp8_meas:
                kernels[f"gemm_N{n}"]["frac_fp8_measured"] = kernels[f"gemm_N{n}"]["TFLOP/s"] / fp8_meas
        # dominant kernel: the block GEMM (sum over the three N per step)
        gemm_ms = sum(k_ms[f"gemm_N{n}"] for n in NS)
        achieved = gemm_flops() / (gemm_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak,
                    "unit": "TFLOP/s", "frac": achieved / fp8_peak,
                    "traffic": gemm_traffic(),
                    "traffic_unit": "bytes per GEMM launch (mean of the step's 3), ncu",
                    "algorithmic_bytes_per_launch": sum(bytes_gemm(M, n) for n in NS) / len(NS),
                    "kernel": "block_gemm_kernel (all three N per step; at N=7168 the call's "
                              "time includes tail_reduce_kernel, which sums the split last wave)",
                    "peak_source": f"{peak_src} bf16 "
                                   f"{'burst' if timed_s < 5.0 else 'sustained'} x {FP8_OVER_BF16} (fp8/bf16 nominal)"}
        if fp8_meas:
            roofline["peak_fp8_measured"] = fp8_meas
            roofline["frac_fp8_measured"] = achieved / fp8_meas
            roofline["peak_fp8_measured_source"] = ("cuBLASLt per-tensor FP8 GEMM (torch._scaled_mm, E4M3, "
                                                    "bf16 out) 8192^3 on random data, best of 10, this process")
        result = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": M, "K": K, "N": list(NS),
                       "parallelism": f"dp{world}" if world > 1 else "none",
                       "l2": "inputs larger than L2 (X 58.7 MB + weights 360 MB per step)"},
            "kernels": kernels,
            "roofline": roofline,
            "e2e": {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        if sharded_ms is not None:
            rows = M * world
            result["per_tensor_sharded"] = {
                "ms": sharded_ms, "rows_total": rows, "K": K,
                "GB/s_total": bytes_per_tensor(rows, K) / (sharded_ms * 1e-3) / 1e9,
                "what": "row-sharded per-tensor quant: local amax, one 4-byte NCCL MAX all-reduce, "
                        "local apply; each rank's X[4096,7168] is its shard; max over ranks"}
        if table is not None:
            result["workloads"] = table
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def single_op(args):
    """--op: one operation at one shape, one JSON line per timing mode."""
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    import fp8_dynamic_quantization_b200 as fq
    fq.library()
    peaks, _ = load_peaks()
    timer = Timer(dev)
    n = args.n or 0
    k = args.k or (2048 if args.op in ("per_tensor", "amax") else 7168)
    for rec in time_op(timer, args.op, args.m, n, k, dev, args.modes.split(","), args.reps,
                       peaks["hbm_gbs"], peaks["bf16_tflops"] * FP8_OVER_BF16):
        print(json.dumps(rec), flush=True)
    if fq.device_status() != 0:
        raise SystemExit("device-side error recorded")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernels", action="store_true",
                    help="skip the per-workload kernel table (and the FP8 peak)")
    ap.add_argument("--op", choices=["per_tensor", "amax", "group128", "group128_ue8m0", "per_channel",
                                     "gemm", "gemm_pt", "gemm_pc", "gemm_ue8m0", "linear"])
    ap.add_argument("--m", type=int)
    ap.add_argument("--n", type=int)
    ap.add_argument("--k", type=int)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--modes", default="cold,graph")
    args = ap.parse_args()
    if args.op:
        single_op(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    result = our_arm(args, rank, world, local_rank)
    if rank == 0 and result is not None:
        if not args.no_cpu_baseline and world == 1:
            x_bits = inputs.bf16_bits(inputs.activations_prefill())
            weights = [inputs.weight_operands(n) for n in NS]
            result["cpu_baseline"] = cpu_baseline(x_bits, weights)
        elif world == 1:
            result["cpu_baseline"] = None
        print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()
