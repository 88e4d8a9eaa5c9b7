"""GPU parity of the per-tensor-scaled FP8 GEMM (the GEMM of the dynamic
per-tensor linear method) against the CPU oracle's definition
Y = s_a * s_b * A * B^T, with the GEMM tolerance the block-scaled tests use."""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
from test_gpu_gemm import assert_within, sample_points, to_dev, y_f64

pytestmark = pytest.mark.gpu


def scalars(seed):
    g = np.random.default_rng(seed)
    return np.float32(g.uniform(1e-3, 1e-1)), np.float32(g.uniform(1e-3, 1e-1))


def run(qa, s_a, qb, s_b, dev):
    return fq.gemm_per_tensor(to_dev(qa, dev), torch.tensor([s_a], device=dev),
                              to_dev(qb, dev), torch.tensor([s_b], device=dev))


@pytest.mark.parametrize("m,n,k", [(1, 8, 128), (3, 200, 256), (16, 300, 1024), (64, 2048, 2048),
                                   (130, 300, 512), (600, 520, 384), (1025, 264, 256)])
def test_per_tensor_gemm_small(oracle_mod, gpu, m, n, k):
    qa, _, qb, _ = inputs.gemm_operands(m, n, k, seed=m + 3 * n + k)
    s_a, s_b = scalars(m + n)
    y = run(qa, s_a, qb, s_b, gpu)
    R, T = oracle_mod.gemm_per_tensor(qa, s_a, qb, s_b)
    assert_within(oracle_mod, y_f64(y), R, T, f"pt {m}x{n}x{k}")
    assert fq.device_status() == 0


@pytest.mark.parametrize("m,n", [(1, 18432), (16, 7168), (64, 2048), (256, 18432), (4096, 7168)])
def test_per_tensor_gemm_full_sizes(oracle_mod, gpu, m, n):
    qa, _, qb, _ = inputs.gemm_operands(m, n, 7168, seed=m + n)
    s_a, s_b = scalars(m * n)
    y = run(qa, s_a, qb, s_b, gpu)
    ms, ns = sample_points(m, n, np.random.default_rng(n))
    sa = np.full((m, 56), s_a, np.float32)
    sb = np.full(((n + 127) // 128, 56), s_b, np.float32)
    R, T = oracle_mod.block_gemm_points(qa, sa, qb, sb, ms, ns)
    assert_within(oracle_mod, y_f64(y)[ms, ns], R, T, f"pt {m}x{n}")


def test_per_tensor_linear_end_to_end(oracle_mod, gpu):
    """bf16 X and W quantised per tensor on the GPU (bit-exact vs the oracle),
    then the per-tensor GEMM."""
    x = inputs.activations_per_tensor(256, k=2048)
    w = inputs.weight_tiny()
    qx, sx = fq.act_quant_per_tensor(x.to(gpu))
    qw, sw = fq.act_quant_per_tensor(w.to(gpu))
    y = fq.gemm_per_tensor(qx, sx, qw, sw)
    rqx, rsx = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    rqw, rsw = oracle_mod.quant_per_tensor(inputs.bf16_bits(w))
    assert np.array_equal(qx.view(torch.uint8).cpu().numpy(), rqx) and np.float32(sx.item()) == rsx
    assert np.array_equal(qw.view(torch.uint8).cpu().numpy(), rqw) and np.float32(sw.item()) == rsw
    R, T = oracle_mod.gemm_per_tensor(rqx, rsx, rqw, rsw)
    assert_within(oracle_mod, y_f64(y), R, T, "per-tensor linear")
    y2 = fq.linear_per_tensor(x.to(gpu), qw, sw)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
