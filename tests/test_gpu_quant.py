"""GPU parity of the quantisation kernels against the CPU oracle.

The bar is bit-exactness: scales compared as fp32 bit patterns, codes as
bytes (NaN codes compared modulo their sign bit, which carries no meaning).
Inputs are the seeded workloads at their full sizes plus edge cases: ragged
and single rows, strided rows, all-zero tensors and groups, signed zeros,
NaN and Inf, and every one of the 65536 bf16 bit patterns.
"""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


def _u8(t):
    return t.view(torch.uint8).cpu().numpy()


def assert_codes_equal(got, want):
    got = np.asarray(got, np.uint8)
    want = np.asarray(want, np.uint8)
    assert got.shape == want.shape
    nan_g = (got & 0x7F) == 0x7F
    nan_w = (want & 0x7F) == 0x7F
    bad = np.flatnonzero((nan_g != nan_w).ravel() | ((got != want) & ~nan_w).ravel())
    assert bad.size == 0, f"{bad.size} codes differ, first at {np.unravel_index(bad[0], got.shape)}: " \
                          f"gpu {got.ravel()[bad[0]]:#04x} oracle {want.ravel()[bad[0]]:#04x}"


def assert_scales_equal(got, want):
    g = np.asarray(got, np.float32).view(np.uint32)
    w = np.asarray(want, np.float32).reshape(g.shape).view(np.uint32)
    nan = np.isnan(np.asarray(want, np.float32).reshape(g.shape))
    assert np.array_equal(np.isnan(np.asarray(got, np.float32)), nan)
    assert np.array_equal(g[~nan], w[~nan])


# ------------------------------------------------------------------ group-128
@pytest.mark.parametrize("m", [1, 32, 4096, 16384])
def test_group128_large_activations(oracle_mod, gpu, m):
    x = inputs.activations_group(m)
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    q, s = fq.act_quant_group128(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)


def test_group128_tiny_layer(oracle_mod, gpu):
    x = inputs.activations_tiny()
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    q, s = fq.act_quant_group128(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)


@pytest.mark.parametrize("m,k", [(1, 128), (3, 128), (7, 384), (33, 1280), (129, 7168)])
def test_group128_ragged(oracle_mod, gpu, m, k):
    x = inputs.activations_group(m, k=k, seed=m * 7 + k)
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    q, s = fq.act_quant_group128(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)


def test_group128_strided_rows(oracle_mod, gpu):
    big = inputs.activations_group(100, k=1024, seed=5)
    view_cpu = big[:, 256:256 + 640]
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(view_cpu))
    view = big.to(gpu)[:, 256:256 + 640]
    assert view.stride(0) == 1024
    q, s = fq.act_quant_group128(view)
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)


# Contiguous tensors take the 4-threads-a-group kernel when x is 32-byte and
# the codes 16-byte aligned, the 8-threads-a-group kernel otherwise: each
# alignment pair is run through the C ABI with buffers placed at that offset.
@pytest.mark.parametrize("x_off,q_off", [(0, 0), (16, 0), (0, 8), (48, 24)])
@pytest.mark.parametrize("m,k", [(33, 1280), (1000, 7168)])
@pytest.mark.parametrize("e8", [False, True])
def test_group128_contiguous_alignments(oracle_mod, gpu, x_off, q_off, m, k, e8):
    lib = fq.library()
    x = inputs.activations_group(m, k=k, seed=m + k + x_off)
    if e8:
        q_ref, s_ref = oracle_mod.quant_group128_ue8m0(inputs.bf16_bits(x))
    else:
        q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    xb = torch.empty(m * k * 2 + 64, dtype=torch.uint8, device=gpu)
    xb[x_off:x_off + m * k * 2].copy_(x.to(gpu).view(torch.uint8).reshape(-1))
    qb = torch.empty(m * k + 64, dtype=torch.uint8, device=gpu)
    g = k // 128
    s = torch.empty(m * g, dtype=torch.uint8 if e8 else torch.float32, device=gpu)
    st = torch.cuda.current_stream().cuda_stream
    fn = lib.fp8_act_quant_group128_ue8m0 if e8 else lib.fp8_act_quant_group128
    assert fn(xb.data_ptr() + x_off, m, k, k, qb.data_ptr() + q_off, k, s.data_ptr(), st) == 0
    torch.cuda.synchronize()
    q = qb[q_off:q_off + m * k].reshape(m, k).cpu().numpy()
    if e8:
        assert np.array_equal(s.cpu().numpy().reshape(m, g), s_ref.reshape(m, g))
    else:
        assert_scales_equal(s.cpu().numpy().reshape(m, g), s_ref)
    assert_codes_equal(q, q_ref)
    assert fq.device_status() == 0


# Seeded random shapes: row counts that leave every possible ragged last
# chunk of the 64-group and 32-group kernels, K from one group to 16, fp32
# and ue8m0 scales, each through the Python binding (aligned buffers).
def test_group128_random_shapes(oracle_mod, gpu):
    g = np.random.default_rng(1234)
    for case in range(24):
        m = int(g.integers(1, 400))
        k = 128 * int(g.integers(1, 17))
        x = inputs.activations_group(m, k=k, seed=7000 + case, dist="normal" if case % 2 else "laplace")
        bits = inputs.bf16_bits(x)
        if case % 3 == 0:
            q, s = fq.act_quant_group128_ue8m0(x.to(gpu))
            q_ref, s_ref = oracle_mod.quant_group128_ue8m0(bits)
            assert np.array_equal(s.cpu().numpy(), np.asarray(s_ref).reshape(m, k // 128)), (m, k)
        else:
            q, s = fq.act_quant_group128(x.to(gpu))
            q_ref, s_ref = oracle_mod.quant_group128(bits)
            assert_scales_equal(s.cpu().numpy(), s_ref)
        assert_codes_equal(_u8(q), q_ref)
    assert fq.device_status() == 0


def test_group128_zero_groups_and_signed_zeros(oracle_mod, gpu):
    x = inputs.activations_group(6, k=512, seed=2)
    x[1, 128:256] = 0.0
    x[2, 0:128] = -0.0
    x[3, :] = 0.0
    x[3, 5] = -0.0
    x[4, 300] = 1e-40          # bf16 subnormal amax
    x[4, 256:300] = 0.0
    x[4, 301:384] = 0.0
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    q, s = fq.act_quant_group128(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)
    assert (s_ref == 0).sum() >= 5


def test_group128_nan_inf(oracle_mod, gpu):
    x = inputs.activations_group(4, k=384, seed=3)
    x[0, 10] = float("nan")
    x[1, 200] = float("inf")
    x[2, 300] = -float("inf")
    x[3, 0] = float("nan")
    x[3, 1] = float("inf")
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    q, s = fq.act_quant_group128(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)


# ------------------------------------------------------------------ per-tensor
@pytest.mark.parametrize("m", [1, 64, 256, 1024, 65536])
def test_per_tensor_sweep(oracle_mod, gpu, m):
    x = inputs.activations_per_tensor(m)
    q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    q, s = fq.act_quant_per_tensor(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
    assert_codes_equal(_u8(q), q_ref)
    assert fq.device_status() == 0


@pytest.mark.parametrize("m,k", [(1, 8), (3, 24), (1, 2048), (2048, 2048), (16384, 2048), (5, 7168), (4096, 7168)])
def test_per_tensor_other_shapes(oracle_mod, gpu, m, k):
    x = inputs.activations_per_tensor(m, k=k, seed=m + k)
    q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    q, s = fq.act_quant_per_tensor(x.to(gpu))
    assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
    assert_codes_equal(_u8(q), q_ref)


# Seeded random shapes across the one-cluster path (small tensors), the
# half-size and full-size amax chunks, and ragged last chunks.
def test_per_tensor_random_shapes(oracle_mod, gpu):
    g = np.random.default_rng(4321)
    for case in range(20):
        m = int(g.integers(1, 3000))
        k = 8 * int(g.integers(1, 400))
        x = inputs.activations_per_tensor(m, k=k, seed=9000 + case)
        q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
        q, s = fq.act_quant_per_tensor(x.to(gpu))
        assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
        assert_codes_equal(_u8(q), q_ref)
    assert fq.device_status() == 0


def test_per_tensor_repeated_calls_reuse_workspace(oracle_mod, gpu):
    """Back-to-back calls of both paths (one cluster, two passes) with one cached workspace."""
    for m in (64, 1024, 1, 300, 65536, 256, 64):
        x = inputs.activations_per_tensor(m, seed=77 + m)
        q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
        q, s = fq.act_quant_per_tensor(x.to(gpu))
        assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
        assert_codes_equal(_u8(q), q_ref)
    assert fq.device_status() == 0


def test_per_tensor_strided_rows(oracle_mod, gpu):
    for m in (8, 4096):
        big = inputs.activations_per_tensor(m, k=4096, seed=m)
        view_cpu = big[:, :2048]
        q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(view_cpu))
        q, s = fq.act_quant_per_tensor(big.to(gpu)[:, :2048])
        assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
        assert_codes_equal(_u8(q), q_ref)


def test_per_tensor_all_zero_and_empty(gpu):
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    x[1, 3] = -0.0
    q, s = fq.act_quant_per_tensor(x.to(gpu))
    assert s.item() == 0.0
    expect = np.where(np.signbit(x.float().numpy()), 0x80, 0x00)
    assert np.array_equal(_u8(q), expect)
    q, s = fq.act_quant_per_tensor(torch.empty(0, 256, dtype=torch.bfloat16, device=gpu))
    assert q.numel() == 0 and s.item() == 0.0


def test_per_tensor_nan_inf(oracle_mod, gpu):
    for val in (float("nan"), float("inf")):
        for m in (4, 65536 // 8):
            x = inputs.activations_per_tensor(m, k=2048, seed=9)
            x[m // 3, 77] = val
            q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
            q, s = fq.act_quant_per_tensor(x.to(gpu))
            assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
            assert_codes_equal(_u8(q), q_ref)


def test_amax_then_apply_matches_per_tensor(oracle_mod, gpu):
    for m in (1, 1024, 65536):
        x = inputs.activations_per_tensor(m).to(gpu)
        word = fq.act_amax(x)
        q1, s1 = fq.act_quant_apply(x, word)
        q2, s2 = fq.act_quant_per_tensor(x)
        bits = inputs.bf16_bits(x.cpu())
        assert word.item() == int((bits & 0x7FFF).max())
        assert torch.equal(s1, s2)
        assert torch.equal(q1.view(torch.uint8), q2.view(torch.uint8))


@pytest.mark.parametrize("amax_value", [448.0, 1.0, 3.0e-38, 1.0e-40, 2.5e38, 7.0, 0.0])
def test_every_bf16_pattern(oracle_mod, gpu, amax_value):
    """All 65536 bf16 bit patterns quantised under a fixed amax word, against
    the oracle's per-element definition (scale = amax/448, code of x/scale)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(512, 128)
    x = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    amax_bits = int(np.float32(amax_value).view(np.uint32) >> 16) & 0x7FFF
    word = torch.tensor([amax_bits], dtype=torch.int32, device=gpu)
    q, s = fq.act_quant_apply(x.to(gpu), word)
    want, s_ref = oracle_mod.quant_apply(bits, amax_bits)
    assert_scales_equal(s.cpu().numpy(), np.array([s_ref]))
    assert_codes_equal(_u8(q), want)


# ------------------------------------------------------------------ weight blocks
@pytest.mark.parametrize("n,k", [(2048, 2048), (200, 384), (128, 128), (1, 256), (300, 7168)])
def test_block128_weight(oracle_mod, gpu, n, k):
    w = inputs.to_bf16(np.random.default_rng(n + k).standard_normal((n, k)))
    if n > 2:
        w[1, 5] = -0.0
    if n > 128 and k >= 256:
        w[128:, 128:256] = 0.0          # an all-zero (ragged) block
    q_ref, s_ref = oracle_mod.quant_block128(inputs.bf16_bits(w))
    q, s = fq.weight_quant_block128(w.to(gpu))
    assert_scales_equal(s.cpu().numpy(), s_ref)
    assert_codes_equal(_u8(q), q_ref)


def test_no_device_errors_recorded(gpu):
    assert fq.device_status(reset=False) == 0


def test_every_x_and_amax_pair(oracle_mod, gpu):
    """Every bf16 value x against every non-negative amax word (2^31 pairs):
    the kernels' division by the scale must give the oracle's codes for all
    of them (including x above the amax, Inf, NaN, zero and subnormal
    scales)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(512, 128)
    x_dev = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(gpu)
    words = torch.arange(0x8000, dtype=torch.int32, device=gpu)
    chunk = 1024
    for w0 in range(0, 0x8000, chunk):
        got = torch.empty(chunk, 512, 128, dtype=torch.uint8, device=gpu)
        scales = torch.empty(chunk, dtype=torch.float32, device=gpu)
        for i in range(chunk):
            q, s = fq.act_quant_apply(x_dev, words[w0 + i:w0 + i + 1])
            got[i] = q.view(torch.uint8)
            scales[i] = s[0]
        got_np = got.cpu().numpy()
        s_np = scales.cpu().numpy()
        for i in range(chunk):
            want, s_ref = oracle_mod.quant_apply(bits, w0 + i)
            if not (np.array_equal(got_np[i], want) and
                    s_np[i].view(np.uint32) == np.float32(s_ref).view(np.uint32)):
                assert_scales_equal(s_np[i:i + 1], np.array([s_ref]))
                assert_codes_equal(got_np[i], want)


def test_empty_inputs_every_quant_entry_point(gpu):
    """Zero rows (and, for the GEMM-side scales, zero weight rows) give empty
    outputs of the right shapes, enqueue nothing that faults, and leave no
    device error."""
    for k in (128, 7168):
        x = torch.empty(0, k, dtype=torch.bfloat16, device=gpu)
        q, s = fq.act_quant_group128(x)
        assert q.shape == (0, k) and s.shape == (0, k // 128)
        q, s = fq.act_quant_group128_ue8m0(x)
        assert q.shape == (0, k) and s.shape == (0, k // 128)
        q, s = fq.act_quant_per_channel(x)
        assert q.shape == (0, k) and s.numel() == 0
        q, s = fq.weight_quant_block128(x)
        assert q.shape == (0, k) and s.numel() == 0
        q, s = fq.weight_quant_block128_ue8m0(x)
        assert q.shape == (0, k) and s.numel() == 0
    assert fq.device_status() == 0
