"""Failure detection without a GPU fault.

A device-side wait that runs out must end the kernel with FP8Q_ERR_TIMEOUT in
the library's status word (read by fp8q_device_status), write no outputs and
leave the context usable.  The GEMM's barrier waits are bounded in SM clock
cycles; FP8Q_WAIT_BUDGET_CYCLES=0 (read once per process, hence a child
process) makes the first wait that is not already satisfied -- the MMA
warp's wait for the first operand tile -- run out.  The kernel then stops
issuing, lets its own copies land, frees its TMEM and returns.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import oracle
import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
dev = torch.device("cuda:0")
fq.device_status(reset=True)
qa, sa, qb, sb = inputs.gemm_operands(4096, 2048, 1024, seed=5)   # one work unit per tile, no split-K
y = torch.full((4096, 2048), 3.0, dtype=torch.bfloat16, device=dev)
fq.block_gemm(torch.from_numpy(qa).to(dev), torch.from_numpy(sa).to(dev),
              torch.from_numpy(qb).to(dev), torch.from_numpy(sb).to(dev), out=y)
assert fq.device_status(reset=True) == 6, "expected FP8Q_ERR_TIMEOUT"
assert bool(torch.all(y == 3.0)), "a timed-out GEMM wrote output"
# the context is still usable: a quantisation call gives the oracle's bytes
x = inputs.activations_group(64, k=1024, seed=3)
q, s = fq.act_quant_group128(x.to(dev))
q_ref, s_ref = oracle.quant_group128(inputs.bf16_bits(x))
assert np.array_equal(q.view(torch.uint8).cpu().numpy(), q_ref)
assert fq.device_status(reset=True) == 0
print("ok")
'''


def test_gemm_wait_timeout_is_reported(gpu, cuda_lib, oracle_mod):
    env = dict(os.environ, FP8Q_WAIT_BUDGET_CYCLES="0")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
