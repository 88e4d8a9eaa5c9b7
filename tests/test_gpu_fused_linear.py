"""GPU parity of the one-call linear (fp8_linear_group128): group-128
quantisation, then the block GEMM launched as its programmatic dependent
(weight loads start before the codes are ready), and the same call with
programmatic dependent launch switched off (FP8Q_PDL=0, read once per
process, hence child processes).  Each is bit-identical to
act_quant_group128 followed by block_gemm, and within the GEMM tolerance of
the oracle's quantisation followed by its block GEMM."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import oracle
import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
from test_gpu_gemm import assert_within, sample_points, to_dev, y_f64
dev = torch.device("cuda:0")
cases = [(1, 300, 128), (5, 2048, 1024), (16, 520, 2048), (17, 2048, 7168), (32, 7168, 7168),
         (33, 1000, 512), (64, 18432, 7168), (200, 600, 2048), (600, 520, 1280)]
for m, n, k in cases:
    x = inputs.activations_group(m, seed=m + n + k, k=k)
    qb, sb = inputs.weight_operands(n, k) if k == 7168 else inputs.gemm_operands(1, n, k, seed=n)[2:]
    tqb = to_dev(qb, dev).view(torch.float8_e4m3fn)
    tsb = to_dev(sb, dev)
    xd = x.to(dev)
    y = fq.linear_fused(xd, tqb, tsb)
    qa_t, sa_t = fq.act_quant_group128(xd)
    y_ref = fq.block_gemm(qa_t, sa_t, tqb, tsb)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), (m, n, k)
    qa, sa = oracle.quant_group128(inputs.bf16_bits(x))
    if m * n <= 600 * 2048:
        R, T = oracle.block_gemm(qa, sa, qb, sb)
        assert_within(oracle, y_f64(y), R, T, f"linear {m}x{n}x{k}")
    else:
        ms, ns = sample_points(m, n, np.random.default_rng(m * n))
        R, T = oracle.block_gemm_points(qa, sa, qb, sb, ms, ns)
        assert_within(oracle, y_f64(y)[ms, ns], R, T, f"linear {m}x{n}x{k}")
# strided tokens with zero, NaN, Inf and signed-zero content
m, n, k = 12, 640, 1024
base = inputs.activations_group(m, seed=3, k=k + 256).clone()
base[2, :] = 0.0
base[3, 5] = float("nan")
base[4, 900] = float("inf")
base[5, 128:256] = -0.0
qb, sb = inputs.gemm_operands(1, n, k, seed=9)[2:]
tqb, tsb = to_dev(qb, dev).view(torch.float8_e4m3fn), to_dev(sb, dev)
xd = base.to(dev)[:, :k]
y = fq.linear_fused(xd, tqb, tsb)
qa_t, sa_t = fq.act_quant_group128(xd)
assert torch.equal(y.view(torch.int16), fq.block_gemm(qa_t, sa_t, tqb, tsb).view(torch.int16))
assert fq.device_status() == 0
print("ok")
'''


@pytest.mark.parametrize("pdl", ["1", "0"])
def test_linear_forms(gpu, cuda_lib, oracle_mod, pdl):
    env = dict(os.environ, FP8Q_PDL=pdl)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
