"""GPU parity of the per-channel path: per-row quantisation bit for bit
against the oracle, and the per-channel-scaled GEMM (row scale of A times
column scale of B in the epilogue) within the GEMM tolerance."""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
from test_gpu_gemm import assert_within, sample_points, to_dev, y_f64
from test_gpu_quant import _u8, assert_codes_equal, assert_scales_equal

pytestmark = pytest.mark.gpu


def check_quant(oracle_mod, x_cpu, gpu, x_dev=None):
    q, s = fq.act_quant_per_channel(x_cpu.to(gpu) if x_dev is None else x_dev)
    rq, rs = oracle_mod.quant_per_channel(inputs.bf16_bits(x_cpu))
    assert_scales_equal(s.cpu().numpy(), rs)
    assert_codes_equal(_u8(q), rq)


@pytest.mark.parametrize("m,k", [(1, 2048), (64, 2048), (4096, 2048), (16, 7168), (4096, 7168),
                                 (3, 8), (5, 24), (33, 1000)])
def test_per_channel_quant(oracle_mod, gpu, m, k):
    check_quant(oracle_mod, inputs.activations_per_tensor(m, k=k), gpu)


def test_per_channel_quant_strided(oracle_mod, gpu):
    base = inputs.activations_per_tensor(50, k=1024)
    check_quant(oracle_mod, base[:, :512].contiguous(), gpu, x_dev=base.to(gpu)[:, :512])


def test_per_channel_quant_special_rows(oracle_mod, gpu):
    rows = np.ones((5, 512), np.float32)
    rows[0] = 0.0
    rows[0, ::2] = -0.0
    rows[1, 7] = np.nan
    rows[2, 100] = -np.inf
    rows[3] = np.float32(2.0 ** -133)
    rows[4, 3] = 3.3e38
    check_quant(oracle_mod, torch.tensor(rows).to(torch.bfloat16), gpu)


def scales(m, n, seed):
    g = np.random.default_rng(seed)
    return g.uniform(1e-3, 1e-1, m).astype(np.float32), g.uniform(1e-3, 1e-1, n).astype(np.float32)


def run(qa, sa, qb, sb, dev):
    return fq.gemm_per_channel(to_dev(qa, dev).view(torch.float8_e4m3fn), to_dev(sa, dev),
                               to_dev(qb, dev).view(torch.float8_e4m3fn), to_dev(sb, dev))


@pytest.mark.parametrize("m,n,k", [(1, 8, 128), (3, 200, 256), (16, 300, 1024), (64, 2048, 2048),
                                   (130, 300, 512), (300, 600, 2048), (600, 520, 384), (1025, 264, 256)])
def test_per_channel_gemm_small(oracle_mod, gpu, m, n, k):
    qa, _, qb, _ = inputs.gemm_operands(m, n, k, seed=m + 5 * n + k)
    sa, sb = scales(m, n, m + n)
    y = run(qa, sa, qb, sb, gpu)
    R, T = oracle_mod.gemm_per_channel(qa, sa, qb, sb)
    assert_within(oracle_mod, y_f64(y), R, T, f"per-channel {m}x{n}x{k}")
    assert fq.device_status() == 0


@pytest.mark.parametrize("m,n", [(1, 18432), (16, 7168), (256, 18432), (4096, 7168)])
def test_per_channel_gemm_full_sizes(oracle_mod, gpu, m, n):
    qa, _, qb, _ = inputs.gemm_operands(m, n, 7168, seed=m + 3 * n)
    sa, sb = scales(m, n, m * 7 + n)
    y = run(qa, sa, qb, sb, gpu)
    ms, ns = sample_points(m, n, np.random.default_rng(n - m))
    ones_a = np.ones((m, 56), np.float32)
    ones_b = np.ones(((n + 127) // 128, 56), np.float32)
    R, T = oracle_mod.block_gemm_points(qa, ones_a, qb, ones_b, ms, ns)
    f = sa.astype(np.float64)[ms] * sb.astype(np.float64)[ns]
    assert_within(oracle_mod, y_f64(y)[ms, ns], R * f, T * f, f"per-channel {m}x{n}")


def test_per_channel_linear_end_to_end(oracle_mod, gpu):
    """X quantised per token and W per output channel on the GPU (bit-exact),
    then the per-channel GEMM."""
    x = inputs.activations_per_tensor(200, k=2048)
    w = inputs.weight_tiny()
    qx, sx = fq.act_quant_per_channel(x.to(gpu))
    qw, sw = fq.act_quant_per_channel(w.to(gpu))
    rqx, rsx = oracle_mod.quant_per_channel(inputs.bf16_bits(x))
    rqw, rsw = oracle_mod.quant_per_channel(inputs.bf16_bits(w))
    assert np.array_equal(_u8(qx), rqx) and np.array_equal(sx.cpu().numpy().view(np.uint32), rsx.view(np.uint32))
    assert np.array_equal(_u8(qw), rqw) and np.array_equal(sw.cpu().numpy().view(np.uint32), rsw.view(np.uint32))
    y = fq.gemm_per_channel(qx, sx, qw, sw)
    R, T = oracle_mod.gemm_per_channel(rqx, rsx, rqw, rsw)
    assert_within(oracle_mod, y_f64(y), R, T, "per-channel linear")
    y2 = fq.linear_per_channel(x.to(gpu), qw, sw)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
