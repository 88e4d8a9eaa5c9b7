"""GPU parity of the ue8m0 (power-of-two scale) quantisation kernels against
the CPU oracle: E8M0 scale bytes and codes compared bit for bit (NaN codes
modulo their sign bit), on the seeded workloads, ragged and strided inputs,
special groups, and every bf16 bit pattern both as a value and as an amax."""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
from test_gpu_quant import _u8, assert_codes_equal

pytestmark = pytest.mark.gpu


def check_group(oracle_mod, x_cpu, gpu):
    q, s = fq.act_quant_group128_ue8m0(x_cpu.to(gpu))
    rq, rs = oracle_mod.quant_group128_ue8m0(inputs.bf16_bits(x_cpu))
    assert np.array_equal(s.cpu().numpy(), rs)
    assert_codes_equal(_u8(q), rq)


@pytest.mark.parametrize("m", [1, 4096, 16384])
def test_group_ue8m0_activations(oracle_mod, gpu, m):
    check_group(oracle_mod, inputs.activations_group(m), gpu)


def test_group_ue8m0_prefill(oracle_mod, gpu):
    check_group(oracle_mod, inputs.activations_prefill(), gpu)


@pytest.mark.parametrize("m,k", [(3, 128), (17, 384), (255, 2048), (1000, 7168)])
def test_group_ue8m0_ragged(oracle_mod, gpu, m, k):
    check_group(oracle_mod, inputs.activations_group(m, seed=m + k, k=k), gpu)


def test_group_ue8m0_strided(oracle_mod, gpu):
    base = inputs.activations_group(64, k=1024)
    xs = base.to(gpu)[:, :768]
    q, s = fq.act_quant_group128_ue8m0(xs)
    rq, rs = oracle_mod.quant_group128_ue8m0(inputs.bf16_bits(base[:, :768]))
    assert np.array_equal(s.cpu().numpy(), rs)
    assert_codes_equal(_u8(q), rq)


def test_group_ue8m0_special_groups(oracle_mod, gpu):
    rows = np.zeros((6, 256), np.float32)
    rows[0, :64] = -0.0
    rows[1] = 1.0; rows[1, 5] = np.nan
    rows[2] = -3.0; rows[2, 200] = -np.inf
    rows[3] = np.float32(2.0 ** -133)
    rows[4] = 448.0; rows[4, 128:] = 450.0
    rows[5, :128] = np.float32(2.0 ** -126); rows[5, 128:] = 3.3e38
    x = torch.tensor(rows).to(torch.bfloat16)
    check_group(oracle_mod, x, gpu)


def test_group_ue8m0_every_bf16_value(oracle_mod, gpu):
    """All 65536 patterns as values: 512 groups of 128 consecutive patterns."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(512, 128)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    check_group(oracle_mod, x, gpu)


def test_group_ue8m0_every_amax(oracle_mod, gpu):
    """Every non-negative bf16 pattern as a group amax (with the rest of the
    group drawn below it), so every exponent decision is exercised."""
    amax = np.arange(0x8000, dtype=np.uint32)
    g = np.random.default_rng(11)
    frac = g.random((0x8000, 127))
    with np.errstate(invalid="ignore"):          # signalling-NaN patterns
        af = (amax << 16).view(np.float32).astype(np.float64)
    rest = np.where(np.isfinite(af)[:, None], af[:, None] * frac * np.where(g.random((0x8000, 127)) < 0.5, -1, 1), 1.0)
    rows = np.concatenate([af[:, None], rest], axis=1).astype(np.float32)
    x = torch.tensor(rows).to(torch.bfloat16)
    check_group(oracle_mod, x, gpu)


@pytest.mark.parametrize("n,k", [(2048, 2048), (300, 7168), (18432, 7168)])
def test_block_ue8m0_weights(oracle_mod, gpu, n, k):
    w = inputs.to_bf16(np.random.default_rng(n + k).standard_normal((n, k)) * 0.02)
    q, s = fq.weight_quant_block128_ue8m0(w.to(gpu))
    rq, rs = oracle_mod.quant_block128_ue8m0(inputs.bf16_bits(w))
    assert np.array_equal(s.cpu().numpy(), rs)
    assert_codes_equal(_u8(q), rq)
