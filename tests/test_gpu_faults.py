"""Failure detection without a GPU fault.

A device-side wait that runs out must end the kernel with FP8Q_ERR_TIMEOUT in
the error word of the stream it was launched on (read by
fp8q_get_last_device_status, or fp8q_device_status for all streams), write no
outputs and leave the context usable.  The GEMM's barrier waits are bounded in SM clock
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


CHILD_STREAMS = r'''
import ctypes, sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import oracle
import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import _abi, inputs
lib = _abi.load()
dev = torch.device("cuda:0")
fq.device_status(reset=True)
# whole tiles, no split-K: the GEMM kernel is the only writer of Y
qa, sa, qb, sb = inputs.gemm_operands(4096, 2048, 1024, seed=7)
ops = [torch.from_numpy(a).to(dev) for a in (qa, sa, qb, sb)]
torch.cuda.synchronize()
sa_, sb_ = torch.cuda.Stream(), torch.cuda.Stream()
ya = torch.full((4096, 2048), 3.0, dtype=torch.bfloat16, device=dev)
yb = torch.full((4096, 2048), 3.0, dtype=torch.bfloat16, device=dev)
lib.fp8q_set_wait_budget_cycles(0)               # stream A's GEMM gives up at its first wait
with torch.cuda.stream(sa_):
    fq.block_gemm(*ops, out=ya)
lib.fp8q_set_wait_budget_cycles(-1)              # the default bound again
with torch.cuda.stream(sb_):
    fq.block_gemm(*ops, out=yb)
assert fq.stream_status(sb_) == 0, "stream B saw stream A's timeout"
assert fq.stream_status(sa_) == 6, "expected FP8Q_ERR_TIMEOUT on stream A"
assert fq.stream_status(sa_) == 0, "reading the status clears it"
assert fq.device_status(reset=True) == 0
assert bool(torch.all(ya == 3.0)), "the timed-out GEMM wrote output"
R, T = oracle.block_gemm(qa, sa, qb, sb)
err = np.abs(yb.float().cpu().numpy().astype(np.float64) - R)
assert np.all(err <= oracle.gemm_tolerance(R, T)), "stream B's GEMM is wrong"
print("ok")
'''


def test_timeout_is_reported_on_its_own_stream(gpu, cuda_lib, oracle_mod):
    """A GEMM on stream A whose waits run out (bound 0) records
    FP8Q_ERR_TIMEOUT in A's error word only: a GEMM launched right after on
    stream B completes correctly, B's status reads FP8Q_OK without waiting
    for A, and reading A's status clears it."""
    r = subprocess.run([sys.executable, "-c", CHILD_STREAMS, ROOT], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
