"""Per-kernel timing sweep over the five workloads (or one op / shape).

    python -m fp8_dynamic_quantization_b200.sweep                 # all workloads
    python -m fp8_dynamic_quantization_b200.sweep --op gemm --m 4096 --n 7168 --k 7168
    python -m fp8_dynamic_quantization_b200.sweep --op group128 --m 16384 --k 7168 --reps 3

Every measurement is the median over `reps` of one call, timed with CUDA
events on the launching stream.  Mode "cold": an L2 flush (a 256 MB read,
which leaves only clean lines in L2) and a GPU sleep run before every call,
outside the timed interval
(the sleep hides the host's launch overhead).  Mode "graph":
`reps` calls captured in one CUDA graph and replayed; time / reps (this is how
the pages timed their amax kernel; inputs that fit in L2 stay L2-warm).
One JSON line per measurement: op, shape, microseconds, algorithmic GB/s
(and TFLOP/s for the GEMM), fraction of the measured HBM / FP8 peaks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import numpy as np
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), 2.0 * float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 2.0 * 1590.0, "fallback"


class Timer:
    def __init__(self, dev):
        self.dev = dev
        self.flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def cold(self, fn, reps):
        fn()                          # untimed: first-call set-up (workspace, tensor maps)
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            # evict the inputs by reading a buffer larger than L2: L2 is left
            # holding clean lines, so the timed call does not also pay for
            # writing back someone else's dirty data
            self.flush_buf.max()
            # keep the GPU busy while the host prepares the call, so host-side
            # overhead never shows up between the two events
            torch.cuda._sleep(200_000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    def graph(self, fn, reps):
        fn()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()                      # populate per-stream workspace caches
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) * 1e3 / reps


def emit(rec):
    print(json.dumps(rec), flush=True)


def run_per_tensor(t, dev, m, k, reps, modes, hbm):
    x = inputs.activations_per_tensor(m, k=k).to(dev)
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.act_quant_per_tensor(x), reps)
        emit({"op": "per_tensor_quant", "M": m, "K": k, "mode": mode, "us": us,
              "GB/s_5B": 5.0 * m * k / us / 1e3, "GB/s_unique_3B": 3.0 * m * k / us / 1e3,
              "frac_hbm_5B": 5.0 * m * k / us / 1e3 / hbm})
        us = getattr(t, mode)(lambda: fq.act_amax(x), reps)
        emit({"op": "amax_only", "M": m, "K": k, "mode": mode, "us": us,
              "GB/s": 2.0 * m * k / us / 1e3, "frac_hbm": 2.0 * m * k / us / 1e3 / hbm})


def run_group(t, dev, m, k, reps, modes, hbm):
    x = inputs.activations_group(m, k=k).to(dev)
    nbytes = 3.0 * m * k + 4.0 * m * (k // 128)
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.act_quant_group128(x), reps)
        emit({"op": "group128_quant", "M": m, "K": k, "mode": mode, "us": us,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_per_channel(t, dev, m, k, reps, modes, hbm):
    x = inputs.activations_per_tensor(m, k=k).to(dev)
    nbytes = 3.0 * m * k + 4.0 * m
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.act_quant_per_channel(x), reps)
        emit({"op": "per_channel_quant", "M": m, "K": k, "mode": mode, "us": us,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_group_ue8m0(t, dev, m, k, reps, modes, hbm):
    x = inputs.activations_group(m, k=k).to(dev)
    nbytes = 3.0 * m * k + m * (k // 128)
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.act_quant_group128_ue8m0(x), reps)
        emit({"op": "group128_quant_ue8m0", "M": m, "K": k, "mode": mode, "us": us,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_gemm_pc(t, dev, m, n, k, reps, modes, hbm, fp8):
    qa, _, qb, _ = inputs.gemm_operands(m, n, k)
    g = np.random.default_rng(m + n)
    tqa = torch.from_numpy(qa).to(dev).view(torch.float8_e4m3fn)
    tqb = torch.from_numpy(qb).to(dev).view(torch.float8_e4m3fn)
    sa = torch.from_numpy(g.uniform(1e-3, 1e-1, m).astype(np.float32)).to(dev)
    sb = torch.from_numpy(g.uniform(1e-3, 1e-1, n).astype(np.float32)).to(dev)
    y = torch.empty(m, (n + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :n]
    nbytes = m * k + n * k + 4.0 * (m + n) + 2.0 * m * n
    flops = 2.0 * m * n * k
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.gemm_per_channel(tqa, sa, tqb, sb, out=y), reps)
        emit({"op": "gemm_per_channel", "M": m, "N": n, "K": k, "mode": mode, "us": us,
              "TFLOP/s": flops / us / 1e6, "frac_fp8": flops / us / 1e6 / fp8,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_linear(t, dev, m, n, k, reps, modes, hbm, fp8):
    """The group-128 linear two ways: quantisation fused into the GEMM, and
    act_quant_group128 followed by block_gemm."""
    x = inputs.activations_group(m, k=k).to(dev)
    qb, sb = inputs.weight_operands(n, k)
    tqb = torch.from_numpy(qb).to(dev).view(torch.float8_e4m3fn)
    tsb = torch.from_numpy(sb).to(dev)
    y = torch.empty(m, (n + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :n]
    nbytes = 2.0 * m * k + n * k + 4.0 * ((n + 127) // 128) * (k // 128) + 2.0 * m * n
    flops = 2.0 * m * n * k

    def two_step():
        qa, sa = fq.act_quant_group128(x)
        fq.block_gemm(qa, sa, tqb, tsb, out=y)
    for mode in modes:
        for name, fn in (("linear_fused", lambda: fq.linear_fused(x, tqb, tsb, out=y)), ("linear_two_step", two_step)):
            us = getattr(t, mode)(fn, reps)
            emit({"op": name, "M": m, "N": n, "K": k, "mode": mode, "us": us,
                  "TFLOP/s": flops / us / 1e6, "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_gemm(t, dev, m, n, k, reps, modes, hbm, fp8):
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k)
    tqa = torch.from_numpy(qa).to(dev).view(torch.float8_e4m3fn)
    tqb = torch.from_numpy(qb).to(dev).view(torch.float8_e4m3fn)
    tsa, tsb = torch.from_numpy(sa).to(dev), torch.from_numpy(sb).to(dev)
    y = torch.empty(m, (n + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :n]
    g = k // 128
    nbytes = m * k + n * k + 4.0 * m * g + 4.0 * ((n + 127) // 128) * g + 2.0 * m * n
    flops = 2.0 * m * n * k
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.block_gemm(tqa, tsa, tqb, tsb, out=y), reps)
        emit({"op": "block_gemm", "M": m, "N": n, "K": k, "mode": mode, "us": us,
              "TFLOP/s": flops / us / 1e6, "frac_fp8": flops / us / 1e6 / fp8,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_gemm_pt(t, dev, m, n, k, reps, modes, hbm, fp8):
    qa, _, qb, _ = inputs.gemm_operands(m, n, k)
    tqa = torch.from_numpy(qa).to(dev).view(torch.float8_e4m3fn)
    tqb = torch.from_numpy(qb).to(dev).view(torch.float8_e4m3fn)
    sa = torch.tensor([0.01], device=dev)
    sb = torch.tensor([0.02], device=dev)
    y = torch.empty(m, (n + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :n]
    nbytes = m * k + n * k + 8.0 + 2.0 * m * n
    flops = 2.0 * m * n * k
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.gemm_per_tensor(tqa, sa, tqb, sb, out=y), reps)
        emit({"op": "gemm_per_tensor", "M": m, "N": n, "K": k, "mode": mode, "us": us,
              "TFLOP/s": flops / us / 1e6, "frac_fp8": flops / us / 1e6 / fp8,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def run_gemm_ue8m0(t, dev, m, n, k, reps, modes, hbm, fp8):
    qa, _, qb, _ = inputs.gemm_operands(m, n, k)
    g = np.random.default_rng(m + n)
    tqa = torch.from_numpy(qa).to(dev).view(torch.float8_e4m3fn)
    tqb = torch.from_numpy(qb).to(dev).view(torch.float8_e4m3fn)
    sa = torch.from_numpy(g.integers(115, 135, (m, k // 128)).astype(np.uint8)).to(dev)
    sb = torch.from_numpy(g.integers(115, 135, ((n + 127) // 128, k // 128)).astype(np.uint8)).to(dev)
    y = torch.empty(m, (n + 7) // 8 * 8, dtype=torch.bfloat16, device=dev)[:, :n]
    nbytes = m * k + n * k + m * k / 128 + ((n + 127) // 128) * k / 128 + 2.0 * m * n
    flops = 2.0 * m * n * k
    for mode in modes:
        us = getattr(t, mode)(lambda: fq.block_gemm_ue8m0(tqa, sa, tqb, sb, out=y), reps)
        emit({"op": "gemm_ue8m0", "M": m, "N": n, "K": k, "mode": mode, "us": us,
              "TFLOP/s": flops / us / 1e6, "frac_fp8": flops / us / 1e6 / fp8,
              "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / hbm})


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["all", "per_tensor", "group128", "gemm", "gemm_pt", "gemm_ue8m0",
                                     "per_channel", "group128_ue8m0", "gemm_pc", "linear"], default="all")
    ap.add_argument("--m", type=int)
    ap.add_argument("--n", type=int)
    ap.add_argument("--k", type=int)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--modes", default="cold,graph")
    a = ap.parse_args()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    hbm, fp8, src = peaks()
    t = Timer(dev)
    modes = a.modes.split(",")
    if a.op == "per_tensor":
        run_per_tensor(t, dev, a.m, a.k or 2048, a.reps, modes, hbm)
    elif a.op == "group128":
        run_group(t, dev, a.m, a.k or 7168, a.reps, modes, hbm)
    elif a.op == "gemm":
        run_gemm(t, dev, a.m, a.n, a.k or 7168, a.reps, modes, hbm, fp8)
    elif a.op == "gemm_pt":
        run_gemm_pt(t, dev, a.m, a.n, a.k or 7168, a.reps, modes, hbm, fp8)
    elif a.op == "gemm_ue8m0":
        run_gemm_ue8m0(t, dev, a.m, a.n, a.k or 7168, a.reps, modes, hbm, fp8)
    elif a.op == "per_channel":
        run_per_channel(t, dev, a.m, a.k or 7168, a.reps, modes, hbm)
    elif a.op == "group128_ue8m0":
        run_group_ue8m0(t, dev, a.m, a.k or 7168, a.reps, modes, hbm)
    elif a.op == "gemm_pc":
        run_gemm_pc(t, dev, a.m, a.n, a.k or 7168, a.reps, modes, hbm, fp8)
    elif a.op == "linear":
        run_linear(t, dev, a.m, a.n, a.k or 7168, a.reps, modes, hbm, fp8)
    else:
        emit({"peaks": {"hbm_gbs": hbm, "fp8_tflops": fp8, "source": src}})
        for m, _, k in inputs.WORKLOAD_SHAPES[2]:
            run_per_tensor(t, dev, m, k, a.reps, modes, hbm)
        for m, _, k in inputs.WORKLOAD_SHAPES[3]:
            run_group(t, dev, m, k, a.reps, modes, hbm)
        run_group(t, dev, 64, 2048, a.reps, modes, hbm)
        for m, n, k in inputs.WORKLOAD_SHAPES[1] + inputs.WORKLOAD_SHAPES[4] + inputs.WORKLOAD_SHAPES[5]:
            run_gemm(t, dev, m, n, k, a.reps, modes, hbm, fp8)
        for m, n, k in inputs.WORKLOAD_SHAPES[4] + inputs.WORKLOAD_SHAPES[5]:
            run_gemm_pt(t, dev, m, n, k, a.reps, modes, hbm, fp8)
        for m, n, k in inputs.WORKLOAD_SHAPES[4] + inputs.WORKLOAD_SHAPES[5]:
            run_gemm_ue8m0(t, dev, m, n, k, a.reps, modes, hbm, fp8)
        for m, n, k in inputs.WORKLOAD_SHAPES[4] + inputs.WORKLOAD_SHAPES[5]:
            run_gemm_pc(t, dev, m, n, k, a.reps, modes, hbm, fp8)
        for m, n, k in inputs.WORKLOAD_SHAPES[4]:
            run_linear(t, dev, m, n, k, a.reps, modes, hbm, fp8)
        for m, _, k in inputs.WORKLOAD_SHAPES[3]:
            run_group_ue8m0(t, dev, m, k, a.reps, modes, hbm)
            run_per_channel(t, dev, m, k, a.reps, modes, hbm)
    if fq.device_status() != 0:
        raise SystemExit("device-side error recorded")


if __name__ == "__main__":
    main()
