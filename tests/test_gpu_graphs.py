"""The library's calls inside a CUDA graph: per-tensor quant, group-128
quant and the block GEMM (CTA-pair tiles with a split last wave) captured
once and replayed on new inputs copied into the captured buffers.  Every
replay must give the bytes of the same calls made directly, and the oracle's
codes and scales.  The per-stream workspaces are created by a first call on
the capture stream, outside the capture (capturing allocates nothing)."""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


def _u8(t):
    return t.view(torch.uint8)


def test_graph_replay_matches_direct_calls(oracle_mod, gpu):
    m, n, k = 1280, 3840, 1024              # CTA pairs; 75 tiles = 74 + 1: a split last wave
    qb_np, sb_np = inputs.weight_operands(n, k, seed=41)
    qb = torch.from_numpy(qb_np).to(gpu).view(torch.float8_e4m3fn)
    sb = torch.from_numpy(sb_np).to(gpu)
    x = torch.empty(m, k, dtype=torch.bfloat16, device=gpu)
    y = torch.empty(m, n, dtype=torch.bfloat16, device=gpu)
    s = torch.cuda.Stream(device=gpu)
    s.wait_stream(torch.cuda.current_stream(gpu))
    with torch.cuda.stream(s):
        x.copy_(inputs.activations_group(m, k=k, seed=40).to(gpu))
        q1, s1 = fq.act_quant_per_tensor(x)      # workspaces for this stream
        q2, s2 = fq.act_quant_group128(x)
        fq.block_gemm(q2, s2, qb, sb, out=y)
    torch.cuda.synchronize(gpu)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        q1, s1 = fq.act_quant_per_tensor(x)
        q2, s2 = fq.act_quant_group128(x)
        fq.block_gemm(q2, s2, qb, sb, out=y)
    for seed in (50, 51, 52):
        xs = inputs.activations_group(m, k=k, seed=seed)
        x.copy_(xs.to(gpu))
        g.replay()
        torch.cuda.synchronize(gpu)
        got = (_u8(q1).clone(), s1.clone(), _u8(q2).clone(), s2.clone(), y.clone())
        d1, e1 = fq.act_quant_per_tensor(x)
        d2, e2 = fq.act_quant_group128(x)
        dy = fq.block_gemm(d2, e2, qb, sb)
        torch.cuda.synchronize(gpu)
        assert torch.equal(got[0], _u8(d1)) and torch.equal(got[1], e1), f"seed {seed}: per-tensor"
        assert torch.equal(got[2], _u8(d2)) and torch.equal(got[3], e2), f"seed {seed}: group-128"
        assert torch.equal(got[4].view(torch.int16), dy.view(torch.int16)), f"seed {seed}: GEMM"
        bits = inputs.bf16_bits(xs)
        rq, rs = oracle_mod.quant_per_tensor(bits)
        assert np.array_equal(got[0].cpu().numpy(), rq) and np.float32(got[1].item()) == rs
        rq2, rs2 = oracle_mod.quant_group128(bits)
        assert np.array_equal(got[2].cpu().numpy(), rq2)
        assert np.array_equal(got[3].cpu().numpy().view(np.uint32), rs2.view(np.uint32))
    del g
    assert fq.device_status() == 0
