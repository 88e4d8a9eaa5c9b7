"""GPU parity of the ue8m0 block-scaled GEMM (E8M0 scales applied by the
tensor cores) against the oracle's definition, with the tolerance of the
fp32-scale GEMM tests: small shapes in full across every launch mode, the
decode and prefill shapes at sampled points, the end-to-end ue8m0 linear
with quantisation checked bit for bit, and NaN scale bytes."""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
from test_gpu_gemm import assert_within, sample_points, to_dev, y_f64

pytestmark = pytest.mark.gpu


def scale_bytes(m, n, k, seed, lo=112, hi=140):
    g = np.random.default_rng(seed)
    return (g.integers(lo, hi, (m, k // 128)).astype(np.uint8),
            g.integers(lo, hi, ((n + 127) // 128, k // 128)).astype(np.uint8))


def run(qa, sa, qb, sb, dev):
    return fq.block_gemm_ue8m0(to_dev(qa, dev).view(torch.float8_e4m3fn), to_dev(sa, dev),
                               to_dev(qb, dev).view(torch.float8_e4m3fn), to_dev(sb, dev))


@pytest.mark.parametrize("m,n,k", [
    (1, 8, 128), (3, 200, 256), (16, 300, 1024), (17, 520, 384), (40, 2048, 2048),
    (100, 256, 7168), (128, 384, 512), (130, 300, 640), (256, 384, 1024), (300, 600, 2048),
    (520, 300, 512), (600, 520, 384), (700, 1000, 1280), (1025, 264, 256),
])
def test_ue8m0_gemm_small_full(oracle_mod, gpu, m, n, k):
    qa, _, qb, _ = inputs.gemm_operands(m, n, k, seed=m * 7 + n + k)
    sa, sb = scale_bytes(m, n, k, m + n + k)
    y = run(qa, sa, qb, sb, gpu)
    R, T = oracle_mod.gemm_ue8m0(qa, sa, qb, sb)
    assert_within(oracle_mod, y_f64(y), R, T, f"ue8m0 {m}x{n}x{k}")
    assert fq.device_status() == 0


@pytest.mark.parametrize("m,n", [(1, 18432), (16, 7168), (64, 18432), (256, 18432), (4096, 7168), (4096, 18432)])
def test_ue8m0_gemm_full_sizes(oracle_mod, gpu, m, n):
    qa, _, qb, _ = inputs.gemm_operands(m, n, 7168, seed=m + 2 * n)
    sa, sb = scale_bytes(m, n, 7168, m * n)
    y = run(qa, sa, qb, sb, gpu)
    ms, ns = sample_points(m, n, np.random.default_rng(n + m))
    R, T = oracle_mod.gemm_ue8m0_points(qa, sa, qb, sb, ms, ns)
    assert_within(oracle_mod, y_f64(y)[ms, ns], R, T, f"ue8m0 {m}x{n}")
    y2 = run(qa, sa, qb, sb, gpu)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))     # deterministic


def test_ue8m0_linear_end_to_end(oracle_mod, gpu):
    """bf16 X and W quantised with ue8m0 scales on the GPU (bit-exact against
    the oracle), then the block-scaled GEMM."""
    x = inputs.activations_group(300, k=2048)
    w = inputs.weight_tiny()
    qx, sx = fq.act_quant_group128_ue8m0(x.to(gpu))
    qw, sw = fq.weight_quant_block128_ue8m0(w.to(gpu))
    rqx, rsx = oracle_mod.quant_group128_ue8m0(inputs.bf16_bits(x))
    rqw, rsw = oracle_mod.quant_block128_ue8m0(inputs.bf16_bits(w))
    assert np.array_equal(qx.view(torch.uint8).cpu().numpy(), rqx) and np.array_equal(sx.cpu().numpy(), rsx)
    assert np.array_equal(qw.view(torch.uint8).cpu().numpy(), rqw) and np.array_equal(sw.cpu().numpy(), rsw)
    y = fq.block_gemm_ue8m0(qx, sx, qw, sw)
    R, T = oracle_mod.gemm_ue8m0(rqx, rsx, rqw, rsw)
    assert_within(oracle_mod, y_f64(y), R, T, "ue8m0 linear")
    y2 = fq.linear_ue8m0(x.to(gpu), qw, sw)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("m", [5, 300])
def test_ue8m0_nan_scale_byte(oracle_mod, gpu, m):
    """Byte 255 (NaN) in one row of A and one weight block: exactly the
    outputs those scales touch are NaN; the rest stay within tolerance."""
    n, k = 400, 512
    qa, _, qb, _ = inputs.gemm_operands(m, n, k, seed=77)
    sa, sb = scale_bytes(m, n, k, 78)
    sa[m // 2, 1] = 255
    sb[2, 3] = 255
    Y = y_f64(run(qa, sa, qb, sb, gpu))
    R, T = oracle_mod.gemm_ue8m0(qa, sa, qb, sb)
    assert np.array_equal(np.isnan(Y), np.isnan(R))
    ok = ~np.isnan(R)
    assert_within(oracle_mod, Y[ok], R[ok], T[ok], "ue8m0 with NaN scales")


def test_ue8m0_extreme_exponents(oracle_mod, gpu):
    """Scales near the ends of the E8M0 range whose products stay finite."""
    m, n, k = 140, 260, 512
    qa, _, qb, _ = inputs.gemm_operands(m, n, k, seed=91)
    g = np.random.default_rng(92)
    sa = np.where(g.random((m, 4)) < 0.5, 10, 240).astype(np.uint8)    # 2^-117 or 2^113
    sb = g.integers(15, 20, ((n + 127) // 128, 4)).astype(np.uint8)        # about 2^-110
    y = run(qa, sa, qb, sb, gpu)
    R, T = oracle_mod.gemm_ue8m0(qa, sa, qb, sb)
    assert_within(oracle_mod, y_f64(y), R, T, "ue8m0 extreme exponents")
