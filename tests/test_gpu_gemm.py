"""GPU parity of the block-scaled FP8 GEMM against the CPU oracle.

Bound (element by element): |Y_gpu - R| <= 2 ulp_bf16(R) + 1e-3 * T, where R
is the oracle's float64 result and T the same sum over |products| with the
scales.  Small shapes are checked everywhere; the full-size decode and
prefill shapes (the launch configurations the benchmark times) at sampled
points -- every corner and tail tile, whole rows and columns, and random
points -- which the oracle evaluates one by one.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def run_gemm(qa, sa, qb, sb, dev, out=None):
    return fq.block_gemm(to_dev(qa, dev).view(torch.float8_e4m3fn), to_dev(sa, dev),
                         to_dev(qb, dev).view(torch.float8_e4m3fn), to_dev(sb, dev), out=out)


def y_f64(y):
    return y.float().cpu().numpy().astype(np.float64)


def assert_within(oracle_mod, Y, R, T, where=""):
    tol = oracle_mod.gemm_tolerance(R, T)
    err = np.abs(Y - R)
    bad = np.flatnonzero(~(err <= tol))
    if bad.size:
        i = bad[np.argmax((err / np.maximum(tol, 1e-300)).ravel()[bad])]
        raise AssertionError(f"{where}: {bad.size} of {err.size} outside tolerance; worst at flat {i}: "
                             f"gpu {Y.ravel()[i]!r} oracle {R.ravel()[i]!r} tol {tol.ravel()[i]!r}")


def sample_points(M, N, g, n_random=4096):
    ms, ns = [], []
    for m in {0, M - 1, M // 2}:
        for n in range(N):
            ms.append(m); ns.append(n)
    for n in {0, N - 1, N // 2, min(N - 1, 129)}:
        for m in range(M):
            ms.append(m); ns.append(n)
    r0 = max(0, M - 128)
    c0 = max(0, N - 128)
    for m in range(r0, M):                   # the last (ragged) 128 x 128 tile
        for n in range(c0, N, 7):
            ms.append(m); ns.append(n)
    ms.extend(g.integers(0, M, n_random).tolist())
    ns.extend(g.integers(0, N, n_random).tolist())
    return np.array(ms, np.int64), np.array(ns, np.int64)


@pytest.mark.parametrize("m,n,k", [
    (1, 8, 128), (1, 128, 128), (3, 200, 256), (16, 300, 1024), (17, 520, 384),
    (40, 2048, 2048), (64, 2048, 2048), (100, 256, 7168), (128, 384, 512),
    (130, 300, 512), (256, 384, 1024), (600, 520, 384), (700, 1000, 1280), (1025, 264, 256),
    # scale rows in 16-byte boxes (K/128 % 4 == 0): ragged M, N past the last
    # weight block, split-K ranges starting inside a group of 4 K blocks
    (300, 600, 2048), (520, 300, 512), (520, 640, 1536), (200, 1100, 3072),
    # CTA-pair tiles (M > 512) with a single K block and with 128 K blocks
    (600, 600, 128), (600, 520, 16384),
])
def test_gemm_small_full(oracle_mod, gpu, m, n, k):
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=m * 131 + n * 7 + k)
    y = run_gemm(qa, sa, qb, sb, gpu)
    R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
    assert_within(oracle_mod, y_f64(y), R, T, f"{m}x{n}x{k}")
    assert fq.device_status() == 0


# Seeded random shapes (N a multiple of 8 for the 16-byte row pitch of Y):
# M up to 1099 and N up to 1272 reach the swapped, single-CTA and CTA-pair
# rows of the launch table, with ragged tiles in both dimensions and a
# range of split-K and split-tail counts.
def test_gemm_random_shapes(oracle_mod, gpu):
    g = np.random.default_rng(2468)
    for case in range(16):
        m = int(g.integers(1, 1100))
        n = 8 * int(g.integers(1, 160))
        k = 128 * int(g.integers(1, 13))
        qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=11000 + case)
        y = run_gemm(qa, sa, qb, sb, gpu)
        R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
        assert_within(oracle_mod, y_f64(y), R, T, f"random {m}x{n}x{k}")
    assert fq.device_status() == 0


@pytest.mark.parametrize("m", [1, 16, 64, 256])
@pytest.mark.parametrize("n", [2048, 7168, 18432])
def test_gemm_decode_shapes(oracle_mod, gpu, m, n):
    qa, sa, qb, sb = inputs.gemm_operands(m, n)
    y = run_gemm(qa, sa, qb, sb, gpu)
    Y = y_f64(y)
    if m == 1:
        R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
        assert_within(oracle_mod, Y, R, T, f"decode {m}x{n}")
    else:
        ms, ns = sample_points(m, n, np.random.default_rng(m + n))
        R, T = oracle_mod.block_gemm_points(qa, sa, qb, sb, ms, ns)
        assert_within(oracle_mod, Y[ms, ns], R, T, f"decode {m}x{n}")
    y2 = run_gemm(qa, sa, qb, sb, gpu)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))     # deterministic


@pytest.mark.parametrize("n", [7168, 18432, 24576])
def test_gemm_prefill_shapes(oracle_mod, gpu, n):
    x = inputs.activations_prefill()
    qa_t, sa_t = fq.act_quant_group128(x.to(gpu))
    qa = qa_t.view(torch.uint8).cpu().numpy()
    sa = sa_t.cpu().numpy()
    q_ref, s_ref = oracle_mod.quant_group128(inputs.bf16_bits(x))
    assert np.array_equal(qa, q_ref) and np.array_equal(sa.view(np.uint32), s_ref.view(np.uint32))
    qb, sb = inputs.weight_operands(n)
    y = fq.block_gemm(qa_t, sa_t, to_dev(qb, gpu), to_dev(sb, gpu))
    ms, ns = sample_points(4096, n, np.random.default_rng(n), n_random=8192)
    R, T = oracle_mod.block_gemm_points(q_ref, s_ref, qb, sb, ms, ns)
    assert_within(oracle_mod, y_f64(y)[ms, ns], R, T, f"prefill 4096x{n}")


def tail_region(M, N, K, sms):
    """Rows and columns of the tiles the launch plan splits along K (the
    tiles past the last full wave, when that wave fills at most half the
    SMs, or half the CTA pairs); empty when no tile is split."""
    plan = (ctypes.c_int * 11)()
    ws = ctypes.c_size_t(0)
    assert fq.library().fp8q_gemm_plan(M, N, K, sms, ctypes.c_size_t(-1).value, plan, ctypes.byref(ws)) == 0
    pair, bn, tiles_p, tiles_q, tail = plan[1], plan[2], plan[5], plan[6], plan[9]
    rows = 256 if pair else 128                 # a CTA pair computes 256-row tiles
    tiles = tiles_p * tiles_q
    out = []
    for t in range(tiles - tail, tiles):
        tp, tq = t % tiles_p, t // tiles_p
        out.append((np.arange(tp * rows, min(M, tp * rows + rows)), np.arange(tq * bn, min(N, tq * bn + bn))))
    return out


def region_points(region):
    ms, ns = [], []
    for rows, cols in region:
        mm, nn = np.meshgrid(rows, cols, indexing="ij")
        ms.append(mm.ravel())
        ns.append(nn.ravel())
    return np.concatenate(ms), np.concatenate(ns)


@pytest.mark.parametrize("m,n,k", [(4096, 7168, 7168), (4000, 7100, 1024)])
def test_gemm_split_tail_tiles(oracle_mod, gpu, m, n, k):
    """Shapes whose tiles leave a short last wave: those tiles run split
    along K and are summed by the tail reduce (launch count 2).  Every output
    of the split tiles (ragged rows and columns in the second shape) and
    sampled points elsewhere against the oracle; two calls give the same
    bytes."""
    sms = torch.cuda.get_device_properties(gpu).multi_processor_count
    region = tail_region(m, n, k, sms)
    assert region, "shape chosen to split its last wave"
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=m + n + k)
    before = fq.library().fp8q_launch_count()
    y = run_gemm(qa, sa, qb, sb, gpu)
    torch.cuda.synchronize()
    assert fq.library().fp8q_launch_count() - before == 2
    Y = y_f64(y)
    ms, ns = region_points(region)
    R, T = oracle_mod.block_gemm_points(qa, sa, qb, sb, ms, ns)
    assert_within(oracle_mod, Y[ms, ns], R, T, f"split tail {m}x{n}x{k}")
    ms, ns = sample_points(m, n, np.random.default_rng(k))
    R, T = oracle_mod.block_gemm_points(qa, sa, qb, sb, ms, ns)
    assert_within(oracle_mod, Y[ms, ns], R, T, f"{m}x{n}x{k}")
    y2 = run_gemm(qa, sa, qb, sb, gpu)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))     # deterministic
    assert fq.device_status() == 0


def test_gemm_tiny_linear_layer_end_to_end(oracle_mod, gpu):
    """bf16 X[64,2048] and W[2048,2048]: GPU quantisation of both, then the
    GEMM, against the oracle's quantisation (bit-exact) and GEMM."""
    x, w = inputs.activations_tiny(), inputs.weight_tiny()
    qx, sx = fq.act_quant_group128(x.to(gpu))
    qw, sw = fq.weight_quant_block128(w.to(gpu))
    y = fq.block_gemm(qx, sx, qw, sw)
    rqx, rsx = oracle_mod.quant_group128(inputs.bf16_bits(x))
    rqw, rsw = oracle_mod.quant_block128(inputs.bf16_bits(w))
    assert np.array_equal(qx.view(torch.uint8).cpu().numpy(), rqx)
    assert np.array_equal(qw.view(torch.uint8).cpu().numpy(), rqw)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), rsw.view(np.uint32))
    R, T = oracle_mod.block_gemm(rqx, rsx, rqw, rsw)
    assert_within(oracle_mod, y_f64(y), R, T, "tiny linear")
    y2 = fq.linear(x.to(gpu), qw, sw)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_gemm_strided_operands_and_output(oracle_mod, gpu):
    m, n, k = 70, 300, 512
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=11)
    a_big = torch.zeros(m, k + 256, dtype=torch.uint8, device=gpu)
    a_big[:, :k] = to_dev(qa, gpu)
    b_big = torch.zeros(n, k + 128, dtype=torch.uint8, device=gpu)
    b_big[:, 128:] = to_dev(qb, gpu)
    out = torch.full((m, n + 28), 7.0, dtype=torch.bfloat16, device=gpu)
    fq.block_gemm(a_big[:, :k], to_dev(sa, gpu), b_big[:, 128:], to_dev(sb, gpu), out=out[:, :n])
    R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
    assert_within(oracle_mod, y_f64(out[:, :n]), R, T, "strided")
    assert torch.all(out[:, n:] == 7.0)                       # nothing written past N


def test_gemm_zero_scales_and_special_codes(oracle_mod, gpu):
    m, n, k = 20, 260, 384
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=5)
    sa[3, :] = 0.0                     # an all-zero activation row
    sa[5, 1] = 0.0                     # one zero group
    sb[2, 0] = 0.0                     # the ragged last weight block, first K block
    qa[7, :] = 0x7E                    # +448 everywhere
    qb[9, :] = 0xFE                    # -448 everywhere
    qa[8, :128] = 0x80                 # -0
    y = run_gemm(qa, sa, qb, sb, gpu)
    R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
    assert_within(oracle_mod, y_f64(y), R, T, "special")
    assert np.all(y_f64(y)[3] == 0)


def test_gemm_empty(gpu):
    qa = torch.empty(0, 256, dtype=torch.uint8, device=gpu)
    sa = torch.empty(0, 2, dtype=torch.float32, device=gpu)
    qb = torch.zeros(64, 256, dtype=torch.uint8, device=gpu)
    sb = torch.ones(1, 2, dtype=torch.float32, device=gpu)
    assert fq.block_gemm(qa, sa, qb, sb).shape == (0, 64)
