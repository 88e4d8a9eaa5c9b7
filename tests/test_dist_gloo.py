"""Host logic of the row-sharded per-tensor path on 2 CPU ranks (gloo).

Each rank holds a slice of the rows; the path takes the local amax word, one
MAX all-reduce of that 4-byte word, then applies the shared scale locally.
On CPU the per-shard compute is done by the oracle (injected through the
amax_fn / apply_fn hooks); the product path uses the CUDA entry points.
The result must equal the oracle's per-tensor quantisation of the whole
tensor, bit for bit, and must also hold when the NaN sits on one rank only.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, case, results):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from fp8_dynamic_quantization_b200 import inputs, per_tensor_sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x = inputs.activations_per_tensor(256, seed=123)
        if case == "nan":
            x[200, 5] = float("nan")          # lands on rank 1 only
        rows = x.shape[0] // world
        shard = x[rank * rows:(rank + 1) * rows]

        def amax_fn(t):
            bits = inputs.bf16_bits(t)
            return torch.tensor([int((bits & 0x7FFF).max())], dtype=torch.int32)

        def apply_fn(t, word):
            return oracle.quant_apply(inputs.bf16_bits(t), int(word.item()))

        q, s = per_tensor_sharded(shard, amax_fn=amax_fn, apply_fn=apply_fn)
        results[rank] = (q, np.float32(s))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["plain", "nan"])
def test_sharded_per_tensor_matches_whole(oracle_mod, case):
    from fp8_dynamic_quantization_b200 import inputs
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(2, _free_port(), case, results), nprocs=2,
                           join=True, start_method="spawn")
        parts = [results[0], results[1]]
    x = inputs.activations_per_tensor(256, seed=123)
    if case == "nan":
        x[200, 5] = float("nan")
    q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    for _, s in parts:
        if np.isnan(s_ref):
            assert np.isnan(s)
        else:
            assert s.view(np.uint32) == np.float32(s_ref).view(np.uint32)
    q = np.concatenate([p[0] for p in parts])
    if case == "nan":
        assert np.all((q & 0x7F) == 0x7F) and np.all((q_ref & 0x7F) == 0x7F)
    else:
        np.testing.assert_array_equal(q, q_ref)
