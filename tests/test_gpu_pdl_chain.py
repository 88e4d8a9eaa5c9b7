"""Back-to-back dependent kernels on one stream.

Every library kernel is launched as a programmatic dependent of the kernel
before it: it may be placed on the GPU while that kernel finishes, and waits
for it before touching global memory.  These tests chain calls where each
kernel reads what the previous one wrote (group quant -> GEMM -> per-tensor
quant of the GEMM's output -> group quant of it), and let torch's caching
allocator hand freed buffers to the next call, so a kernel that started
reading or writing early would see stale inputs or clobber live ones.  Every
result is compared with the oracle run on the GPU's own intermediate values.
"""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


def _u8(t):
    return t.view(torch.uint8).cpu().numpy()


def test_dependent_chain_matches_the_oracle(oracle_mod, gpu):
    m, n, k = 384, 2048, 1024
    w = inputs.to_bf16(inputs.rng(71).standard_normal((n, k)))
    qb, sb = fq.weight_quant_block128(w.to(gpu))            # kernel 1
    qb_h, sb_h = _u8(qb), sb.cpu().numpy()
    for it in range(4):
        x = inputs.activations_group(m, k=k, seed=700 + it).to(gpu)
        qa, sa = fq.act_quant_group128(x)                     # reads x
        y = fq.block_gemm(qa, sa, qb, sb)                     # reads qa, sa
        q2, s2 = fq.act_quant_per_tensor(y)                   # reads y
        q3, s3 = fq.act_quant_group128(y)                     # reads y again
        qa_h, sa_h = _u8(qa), sa.cpu().numpy()
        y_bits = inputs.bf16_bits(y.cpu())
        rqa, rsa = oracle_mod.quant_group128(inputs.bf16_bits(x.cpu()))
        assert np.array_equal(qa_h, rqa) and np.array_equal(sa_h.view(np.uint32), rsa.view(np.uint32))
        R, T = oracle_mod.block_gemm(rqa, rsa, qb_h, sb_h)
        Y = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(Y - R) <= oracle_mod.gemm_tolerance(R, T)), f"iteration {it}: GEMM"
        rq2, rs2 = oracle_mod.quant_per_tensor(y_bits)
        assert np.float32(s2.item()) == rs2 and np.array_equal(_u8(q2), rq2), f"iteration {it}: per-tensor of Y"
        rq3, rs3 = oracle_mod.quant_group128(y_bits)
        assert np.array_equal(_u8(q3), rq3) and np.array_equal(s3.cpu().numpy().view(np.uint32),
                                                               rs3.view(np.uint32)), f"iteration {it}: group of Y"
        del x, qa, sa, y, q2, s2, q3, s3                     # buffers go back to the allocator
    assert fq.device_status() == 0


def test_outputs_overwritten_in_stream_order(oracle_mod, gpu):
    """The same output buffer written by consecutive GEMMs of different
    inputs, and read by a quantisation between them: each reader sees the
    write just before it, never the next one."""
    m, n, k = 256, 1024, 512
    qa1, sa1, qb, sb = inputs.gemm_operands(m, n, k, seed=81)
    qa2, sa2, _, _ = inputs.gemm_operands(m, n, k, seed=82)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(gpu)
    y = torch.empty(m, n, dtype=torch.bfloat16, device=gpu)
    fq.block_gemm(d(qa1), d(sa1), d(qb), d(sb), out=y)
    q1, s1 = fq.act_quant_per_tensor(y)
    fq.block_gemm(d(qa2), d(sa2), d(qb), d(sb), out=y)
    q2, s2 = fq.act_quant_per_tensor(y)
    torch.cuda.synchronize()
    R1, T1 = oracle_mod.block_gemm(qa1, sa1, qb, sb)
    R2, T2 = oracle_mod.block_gemm(qa2, sa2, qb, sb)
    Y2 = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Y2 - R2) <= oracle_mod.gemm_tolerance(R2, T2))
    rq2, rs2 = oracle_mod.quant_per_tensor(inputs.bf16_bits(y.cpu()))
    assert np.float32(s2.item()) == rs2 and np.array_equal(_u8(q2), rq2)
    # the first quantisation saw the first GEMM's Y: its scale is that
    # tensor's amax / 448, and the GPU's Y1 is within the GEMM tolerance of R1
    amax1 = float(np.abs(R1).max())
    tol1 = float(oracle_mod.gemm_tolerance(R1, T1).max())
    assert abs(float(s1.item()) * 448.0 - amax1) <= tol1 + 1e-6 * amax1
    assert fq.device_status() == 0
