"""The row-sharded per-tensor path on the GPU through NCCL: local amax word
(fp8_act_amax), one 4-byte MAX all-reduce, local apply (fp8_act_quant_apply).

A single-rank NCCL group on cuda:0 runs the product path end to end -- the
device amax word goes through NCCL's all-reduce and back into the apply
kernel -- and must equal the oracle's per-tensor quantisation of the tensor
bit for bit.  Ranks on several GPUs are covered by the same host logic on
CPU ranks (gloo) in test_dist_gloo.py; more than one rank per GPU is not run.
"""
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import datetime, os, sys
import numpy as np, torch
import torch.distributed as dist
sys.path.insert(0, sys.argv[1])
import oracle
import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
dev = torch.device("cuda:0")
torch.cuda.set_device(dev)
os.environ["MASTER_ADDR"] = "127.0.0.1"
os.environ["MASTER_PORT"] = sys.argv[2]
dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60), device_id=dev)
try:
    for m, k, nan in [(4096, 7168, False), (300, 2048, True), (1, 8, False)]:
        x = inputs.activations_per_tensor(m, k=k, seed=m + k)
        if nan:
            x[m // 2, 3] = float("nan")
        q, s = fq.per_tensor_sharded(x.to(dev))
        rq, rs = oracle.quant_per_tensor(inputs.bf16_bits(x))
        a, b = np.float32(s.item()), np.float32(rs)
        assert (np.isnan(a) and np.isnan(b)) or a.view(np.uint32) == b.view(np.uint32), (m, k)
        assert np.array_equal(q.view(torch.uint8).cpu().numpy(), rq), (m, k)
    assert fq.device_status() == 0
finally:
    dist.destroy_process_group()
print("ok")
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_sharded_per_tensor_through_nccl(gpu, cuda_lib, oracle_mod):
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, str(_free_port())], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
