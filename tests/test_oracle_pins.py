"""Pins for the CPU oracle: each check compares it with something other than
itself -- the E4M3 format definition, torch's own float8 conversion (an
independent library routine), closed forms, float64 brute force and
invariants -- chosen so that a dropped term, a wrong sign, index or tie rule,
or a transposed operand fails at least one of them.

Sources: "How to Profile DeepSeek-V3 Inference Kernels Using Triton
Autotuning" (block-wise activation quant; FP8 GEMM with per-block scaling,
BLOCK_K = 128); "Size the per-tensor FP8 dynamic-quant amax grid to the
input" (exact amax, scale = amax / 448, bitwise-identical bytes; strided
inputs and NaN parity from the review); "The Surgical Precision Flip ..."
(Assumptions and Their Validity: E4M3 is 1/4/3 bits and widens to bf16
losslessly).
"""
import numpy as np
import pytest
import torch

from fp8_dynamic_quantization_b200 import inputs

F8 = torch.float8_e4m3fn


def torch_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(F8).to(torch.float64).numpy()


def torch_encode(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    return t.to(F8).view(torch.uint8).numpy()


ALL_CODES = np.arange(256, dtype=np.uint8)
FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


# ------------------------------------------------------------------ decode
def test_decode_enumerates_format(oracle_mod):
    v = oracle_mod.e4m3_decode(ALL_CODES)
    nan = np.isnan(v)
    assert sorted(np.flatnonzero(nan).tolist()) == [0x7F, 0xFF]
    fin = v[~nan]
    assert fin.size == 254
    assert np.unique(fin).size == 253                 # +0 and -0 coincide
    assert fin.max() == 448.0 and fin.min() == -448.0
    pos = fin[fin > 0]
    assert pos.min() == 2.0 ** -9                      # smallest subnormal
    assert oracle_mod.e4m3_decode(0x08) == 2.0 ** -6   # smallest normal
    assert oracle_mod.e4m3_decode(0x38) == 1.0         # exponent bias 7
    assert np.signbit(oracle_mod.e4m3_decode(0x80))
    # sign bit is bit 7
    np.testing.assert_array_equal(v[0x80:][~nan[0x80:]], -v[:0x80][~nan[:0x80]])


def test_decode_matches_torch(oracle_mod):
    ours = oracle_mod.e4m3_decode(ALL_CODES)
    ref = torch_decode(ALL_CODES)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    m = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[m], ref[m])
    np.testing.assert_array_equal(np.signbit(ours[m]), np.signbit(ref[m]))


def test_e4m3_widens_to_bf16_losslessly(oracle_mod):
    v = oracle_mod.e4m3_decode(FINITE)
    back = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(back, v)


# ------------------------------------------------------------------ encode
def test_encode_inverts_decode(oracle_mod):
    v = oracle_mod.e4m3_decode(FINITE).astype(np.float32)
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(v), FINITE)


def test_encode_special_values(oracle_mod):
    cases = [
        (448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (1e30, 0x7E), (np.inf, 0x7E),
        (-448.0, 0xFE), (-np.inf, 0xFE), (-1e30, 0xFE),
        (0.0, 0x00), (-0.0, 0x80), (2.0 ** -10, 0x00), (-(2.0 ** -10), 0x80),
        (1.5 * 2.0 ** -10, 0x01), (-(1e-30), 0x80), (2.0 ** -6, 0x08),
        (1.0625, 0x38),      # tie between 1.0 and 1.125 -> even mantissa 0
        (1.1875, 0x3A),      # tie between 1.125 and 1.25 -> even mantissa 2
        (432.0, 0x7E),       # tie between 416 and 448 -> even mantissa 6
        (float(np.float32(1.0625) + np.float32(2.0 ** -20)), 0x39),
    ]
    vals = np.array([c[0] for c in cases], dtype=np.float32)
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(vals),
                                  np.array([c[1] for c in cases], dtype=np.uint8))
    nan_codes = oracle_mod.e4m3_encode(np.array([np.nan, -np.nan], np.float32))
    assert all((c & 0x7F) == 0x7F for c in nan_codes)


def _check_range_vs_torch(oracle_mod, first, count, sign):
    bits = (np.arange(first, first + count, dtype=np.uint64) | sign).astype(np.uint32)
    ours = oracle_mod.e4m3_encode_range(int(bits[0]), count)
    ref = torch_encode(bits.view(np.float32))
    bad = np.flatnonzero(ours != ref)
    assert bad.size == 0, (hex(int(bits[bad[0]])), ours[bad[0]], ref[bad[0]])


@pytest.mark.slow
def test_encode_exhaustive_vs_torch(oracle_mod):
    """Every fp32 bit pattern with |v| <= 464, both signs, against torch's
    float8_e4m3fn conversion (RNE; it agrees with saturation up to 464 and
    returns NaN above, where ours saturates by definition)."""
    limit = 0x43E80001                       # up to and including 464.0
    chunk = 1 << 24
    for sign in (0, 0x80000000):
        for first in range(0, limit, chunk):
            _check_range_vs_torch(oracle_mod, first, min(chunk, limit - first), sign)


def test_encode_nearest_by_brute_force(oracle_mod):
    """Nearest representable value, ties to the even code, by enumeration."""
    mags = oracle_mod.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))   # 127 magnitudes
    g = np.random.default_rng(7)
    mids = (mags[1:] + mags[:-1]) / 2.0
    mids32 = mids.astype(np.float32)
    assert np.all(mids32.astype(np.float64) == mids)                     # exact
    around = np.concatenate([mids32, np.nextafter(mids32, np.float32(0)),
                             np.nextafter(mids32, np.float32(np.inf))])
    rand = (np.exp2(g.uniform(-14, 9, 200000)) * g.uniform(1, 2, 200000)).astype(np.float32)
    v = np.concatenate([around, rand, mags.astype(np.float32)])
    v = v[v < 448]
    d = np.abs(v.astype(np.float64)[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    idx = np.where(cand.sum(1) == 2,
                   np.argmax(cand & (np.arange(127) % 2 == 0)[None, :], axis=1),
                   np.argmax(cand, axis=1))
    expect = idx.astype(np.uint8)        # code == index for magnitudes 0x00..0x7E
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(v), expect)
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(-v), expect | 0x80)


def test_encode_monotone(oracle_mod):
    g = np.random.default_rng(3)
    v = np.sort(np.concatenate([g.standard_normal(100000) * 100,
                                g.standard_normal(10000) * 1e-2])).astype(np.float32)
    dec = oracle_mod.e4m3_decode(oracle_mod.e4m3_encode(v))
    assert np.all(np.diff(dec) >= 0)


# ------------------------------------------------------------------ scale
def test_scale_closed_form(oracle_mod):
    assert oracle_mod.scale_from_amax(448.0) == 1.0
    for k in range(-20, 21):
        assert oracle_mod.scale_from_amax(448.0 * 2.0 ** k) == np.float32(2.0 ** k)
    assert oracle_mod.scale_from_amax(0.0) == 0.0
    assert np.isnan(oracle_mod.scale_from_amax(np.nan))
    g = np.random.default_rng(11)
    a = (np.exp2(g.uniform(-30, 30, 1000))).astype(np.float32)
    ours = np.array([oracle_mod.scale_from_amax(x) for x in a], dtype=np.float32)
    ref = (torch.from_numpy(a) / torch.tensor(448.0, dtype=torch.float32)).numpy()
    np.testing.assert_array_equal(ours, ref)


# ------------------------------------------------------------------ per-tensor
def torch_quant(xf32: torch.Tensor, s: float) -> np.ndarray:
    """Codes by torch: IEEE fp32 division then torch's float8 conversion
    (saturation applied first, since torch maps large values to NaN)."""
    q = xf32 / torch.tensor(s, dtype=torch.float32)
    q = torch.clamp(q, -448.0, 448.0)
    return q.to(F8).view(torch.uint8).numpy()


def test_per_tensor_unit_scale_is_plain_conversion(oracle_mod):
    x = inputs.activations_per_tensor(64)
    xf = x.float()
    xf = xf / xf.abs().max() * 448.0          # amax becomes exactly 448
    xb = xf.to(torch.bfloat16)
    assert xb.float().abs().max().item() == 448.0
    q, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(xb))
    assert s == 1.0
    np.testing.assert_array_equal(q, xb.float().to(F8).view(torch.uint8).numpy())


@pytest.mark.parametrize("m", [1, 64, 256])
def test_per_tensor_matches_torch(oracle_mod, m):
    x = inputs.activations_per_tensor(m)
    q, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    amax = x.float().abs().max()
    assert s == (amax / torch.tensor(448.0)).item()
    np.testing.assert_array_equal(q, torch_quant(x.float(), s))


def test_per_tensor_zero_convention(oracle_mod):
    x = torch.zeros(3, 256, dtype=torch.bfloat16)
    x[1, 5] = -0.0
    x[2, :] = -0.0
    q, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    assert s == 0.0
    expect = np.where(np.signbit(x.float().numpy()), 0x80, 0x00).astype(np.uint8)
    np.testing.assert_array_equal(q, expect)


def test_per_tensor_nan_and_inf(oracle_mod):
    x = inputs.activations_per_tensor(4, k=256)
    xn = x.clone()
    xn[2, 17] = float("nan")
    q, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(xn))
    assert np.isnan(s)
    assert np.all((q & 0x7F) == 0x7F)
    xi = x.clone()
    xi[1, 3] = float("inf")
    q, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(xi))
    assert np.isinf(s)
    fin = np.isfinite(xi.float().numpy())
    assert np.all((q[fin] & 0x7F) == 0)                 # x / inf = +-0
    assert (q[1, 3] & 0x7F) == 0x7F                    # inf / inf = NaN


def test_per_tensor_round_trip_bound(oracle_mod):
    x = inputs.activations_per_tensor(256)
    q, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    xv = x.float().numpy().astype(np.float64)
    dq = oracle_mod.e4m3_decode(q) * float(s)
    r = np.abs(xv / float(s))
    e = np.floor(np.log2(np.maximum(r, 2.0 ** -6)))
    half_ulp = np.ldexp(1.0, (e - 4).astype(np.int64))      # 1/2 * 2^(e-3)
    slack = 2.0 * np.abs(xv) * 2.0 ** -23
    assert np.all(np.abs(dq - xv) <= half_ulp * float(s) + slack)
    i = np.unravel_index(np.argmax(np.abs(xv)), xv.shape)
    assert abs(abs(dq[i]) - float(np.abs(xv).max())) <= float(s) * 16   # amax element ~ 448*s


def test_per_tensor_permutation_invariant(oracle_mod):
    x = inputs.activations_per_tensor(64)
    _, s = oracle_mod.quant_per_tensor(inputs.bf16_bits(x))
    perm = torch.randperm(x.numel(), generator=torch.Generator().manual_seed(5))
    xp = x.reshape(-1)[perm].reshape(x.shape).contiguous()
    qp, sp = oracle_mod.quant_per_tensor(inputs.bf16_bits(xp))
    assert sp == s


def test_per_tensor_strided_rows(oracle_mod):
    big = inputs.activations_per_tensor(32, k=512)
    view = big[:, :256]                                  # row stride 512
    q1, s1 = oracle_mod.quant_per_tensor(inputs.bf16_bits(view))
    q2, s2 = oracle_mod.quant_per_tensor(inputs.bf16_bits(view.contiguous()))
    assert s1 == s2
    np.testing.assert_array_equal(q1, q2)
    assert s1 == (view.float().abs().max() / 448.0).item()


# ------------------------------------------------------------------ groups
def torch_group_quant(x: torch.Tensor, rows: int, cols: int):
    """Block quant by torch ops: amax over (rows x cols) blocks, fp32
    division by 448, torch's float8 conversion."""
    xf = x.float()
    M, K = xf.shape
    Mp = -(-M // rows) * rows
    pad = torch.zeros(Mp, K)
    pad[:M] = xf.abs()
    amax = pad.reshape(Mp // rows, rows, K // cols, cols).amax(dim=(1, 3))
    s = amax / torch.tensor(448.0)
    s_full = s.repeat_interleave(rows, 0)[:M].repeat_interleave(cols, 1)
    safe = torch.where(s_full == 0, torch.ones_like(s_full), s_full)
    q = torch.clamp(xf / safe, -448, 448).to(F8).view(torch.uint8)
    zero_code = torch.where(torch.signbit(xf), 0x80, 0x00).to(torch.uint8)
    q = torch.where(s_full == 0, zero_code, q)
    return q.numpy(), s.numpy()


@pytest.mark.parametrize("m,k", [(1, 7168), (32, 7168), (5, 256)])
def test_group128_matches_torch(oracle_mod, m, k):
    x = inputs.activations_group(m, k=k)
    q, s = oracle_mod.quant_group128(inputs.bf16_bits(x))
    qr, sr = torch_group_quant(x, 1, 128)
    np.testing.assert_array_equal(s, sr)
    np.testing.assert_array_equal(q, qr)


def test_group128_zero_group(oracle_mod):
    x = inputs.activations_per_tensor(64)          # row 32 holds one zero group
    q, s = oracle_mod.quant_group128(inputs.bf16_bits(x))
    zr, zg = np.argwhere(s == 0)[0]
    assert zr == 32
    assert np.all(q[zr, 128 * zg:128 * zg + 128] == 0)
    qr, sr = torch_group_quant(x, 1, 128)
    np.testing.assert_array_equal(q, qr)
    np.testing.assert_array_equal(s, sr)


def test_group128_strided(oracle_mod):
    big = inputs.activations_group(8, k=1024)
    view = big[:, 128:640]
    q1, s1 = oracle_mod.quant_group128(inputs.bf16_bits(view))
    q2, s2 = oracle_mod.quant_group128(inputs.bf16_bits(view.contiguous()))
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s1, s2)


@pytest.mark.parametrize("n", [256, 200])
def test_block128_matches_torch(oracle_mod, n):
    w = inputs.to_bf16(np.random.default_rng(n).standard_normal((n, 384)))
    q, s = oracle_mod.quant_block128(inputs.bf16_bits(w))
    qr, sr = torch_group_quant(w, 128, 128)
    np.testing.assert_array_equal(s, sr)
    np.testing.assert_array_equal(q, qr)


# ------------------------------------------------------------------ GEMM
def torch_block_gemm(qa, sa, qb, sb):
    """float64 via torch: dequantised per-128 block products, scaled, summed."""
    A = torch.from_numpy(torch_decode(qa))
    B = torch.from_numpy(torch_decode(qb))
    M, K = A.shape
    N = B.shape[0]
    out = torch.zeros(M, N, dtype=torch.float64)
    sbn = torch.from_numpy(sb.astype(np.float64)).repeat_interleave(128, 0)[:N]
    for kb in range(K // 128):
        p = A[:, kb * 128:(kb + 1) * 128] @ B[:, kb * 128:(kb + 1) * 128].T
        out += torch.from_numpy(sa[:, kb].astype(np.float64))[:, None] * sbn[None, :, kb] * p
    return out.numpy()


@pytest.mark.parametrize("m,n,k", [(1, 8, 128), (5, 7, 256), (8, 200, 384), (3, 130, 128)])
def test_gemm_matches_float64_brute_force(oracle_mod, m, n, k):
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=m * 1000 + n)
    R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
    ref = torch_block_gemm(qa, sa, qb, sb)
    np.testing.assert_allclose(R, ref, rtol=1e-12, atol=1e-300)
    assert np.all(T >= np.abs(R) * (1 - 1e-12))


def test_gemm_exact_integer_case(oracle_mod):
    """Unit scales and codes for {0, +-1, +-2}: an exact integer matmul."""
    g = np.random.default_rng(2)
    vals = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)   # 0, 1, -1, 2, -2
    qa = vals[g.integers(0, 5, (9, 256))]
    qb = vals[g.integers(0, 5, (300, 256))]
    sa = np.ones((9, 2), np.float32)
    sb = np.ones((3, 2), np.float32)
    R, _ = oracle_mod.block_gemm(qa, sa, qb, sb)
    ia = torch.from_numpy(torch_decode(qa)).to(torch.int64)
    ib = torch.from_numpy(torch_decode(qb)).to(torch.int64)
    np.testing.assert_array_equal(R, (ia @ ib.T).numpy().astype(np.float64))
    bf = oracle_mod.f64_to_bf16(R)
    ref = torch.from_numpy(R).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bf, ref)


def test_gemm_single_block_and_linearity(oracle_mod):
    qa, sa, qb, sb = inputs.gemm_operands(4, 256, 512, seed=9)
    R, _ = oracle_mod.block_gemm(qa, sa, qb, sb)
    j = 2
    only = sa.copy()
    only[:, [i for i in range(4) if i != j]] = 0
    Rj, _ = oracle_mod.block_gemm(qa, only, qb, sb)
    A = torch_decode(qa[:, 128 * j:128 * j + 128])
    B = torch_decode(qb[:, 128 * j:128 * j + 128])
    sbn = np.repeat(sb[:, j].astype(np.float64), 128)[:256]
    np.testing.assert_allclose(Rj, sa[:, j, None].astype(np.float64) * sbn[None, :] * (A @ B.T),
                               rtol=1e-14)
    doubled = sa.copy()
    doubled[:, j] *= 2
    R2, _ = oracle_mod.block_gemm(qa, doubled, qb, sb)
    np.testing.assert_allclose(R2 - R, Rj, rtol=1e-9, atol=1e-12 * np.abs(R).max())


def test_gemm_scale_index_uses_row_block_of_b(oracle_mod):
    """Rows n and n+128 of B use different sb rows; rows within a block share one."""
    qa, sa, qb, sb = inputs.gemm_operands(2, 256, 128, seed=4)
    qb[128:] = qb[:128]
    sb2 = sb.copy()
    sb2[1] = sb[0] * 4
    R, _ = oracle_mod.block_gemm(qa, sa, qb, sb2)
    np.testing.assert_allclose(R[:, 128:], 4 * R[:, :128], rtol=1e-14)


def test_gemm_points_equal_full(oracle_mod):
    qa, sa, qb, sb = inputs.gemm_operands(6, 300, 256, seed=1)
    R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
    g = np.random.default_rng(0)
    ms, ns = g.integers(0, 6, 50), g.integers(0, 300, 50)
    Rp, Tp = oracle_mod.block_gemm_points(qa, sa, qb, sb, ms, ns)
    np.testing.assert_array_equal(Rp, R[ms, ns])
    np.testing.assert_array_equal(Tp, T[ms, ns])


def test_gemm_strided_operands(oracle_mod):
    qa, sa, qb, sb = inputs.gemm_operands(4, 64, 256, seed=3)
    wide = np.zeros((64, 512), np.uint8)
    wide[:, :256] = qb
    R1, _ = oracle_mod.block_gemm(qa, sa, qb, sb)
    R2, _ = oracle_mod.block_gemm(qa, sa, wide[:, :256], sb)
    np.testing.assert_array_equal(R1, R2)


def test_f64_to_bf16_matches_torch(oracle_mod):
    g = np.random.default_rng(1)
    v = np.concatenate([g.standard_normal(100000) * 10.0 ** g.integers(-40, 38, 100000),
                        [0.0, -0.0, 1e-45, -1e-45, 3.4e38, -3.4e38]]).astype(np.float32)
    ours = oracle_mod.f64_to_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def _bf16_rne_exact(v: float) -> int:
    """bf16 bit pattern of the float64 value v rounded once, to nearest with
    ties to even, computed with exact rationals: the float64 value as a
    Fraction, its bf16 quantum (8 significant bits, normal range from
    2^-126, subnormal quantum 2^-133), round(n) on the exact quotient
    (Python rounds a Fraction half to even), overflow to infinity."""
    import math
    import struct
    from fractions import Fraction
    sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
    a = Fraction(abs(v))
    if a == 0:
        return sign
    k = math.frexp(abs(v))[1] - 1                  # floor(log2 |v|)
    quantum = Fraction(2) ** (max(k, -126) - 7)
    r = round(a / quantum) * quantum
    if r >= Fraction(2) ** 128:
        return sign | 0x7F80
    return sign | (struct.unpack("<I", struct.pack("<f", float(r)))[0] >> 16)


def _bf16_value(bits: int) -> float:
    import struct
    return struct.unpack("<f", struct.pack("<I", bits << 16))[0]


def test_f64_to_bf16_rounds_float64_values_once(oracle_mod):
    """Float64 values that fp32 cannot hold: the exact midpoints between
    neighbouring bf16 values, one float64 ulp either side of them, values a
    hair above a midpoint whose fp32 rounding lands on the midpoint (rounding
    through fp32 first would then tie to even and go the wrong way),
    subnormal and overflow boundaries, and random full-precision values --
    against a one-rounding reference built from exact rationals.  A
    double-rounding variant (float64 -> fp32 -> bf16) is checked to fail on
    these cases, so the pin would catch that mistake."""
    import math
    g = np.random.default_rng(11)
    vals = []
    lo_bits = g.integers(0x0001, 0x7F7F, 400)                      # finite, nonzero bf16
    for b in list(lo_bits) + [0x0001, 0x007F, 0x0080, 0x3F80, 0x7F7E]:
        lo, hi = _bf16_value(int(b)), _bf16_value(int(b) + 1)
        mid = (lo + hi) / 2.0                                        # exact in float64
        vals += [mid, math.nextafter(mid, math.inf), math.nextafter(mid, -math.inf)]
        # just above the midpoint by less than half an fp32 ulp of it
        vals.append(mid + math.ulp(mid) * 64.0)
        vals.append(mid - math.ulp(mid) * 64.0)
    top = _bf16_value(0x7F7F)
    vals += [top + math.ulp(top) * (2.0 ** 44), 2.0 ** 128 - 2.0 ** 119,
             math.nextafter(2.0 ** 128 - 2.0 ** 119, 0.0), 2.0 ** -134, math.nextafter(2.0 ** -134, 1.0),
             5e-324, 1e-300, 3 * 2.0 ** -135]
    vals += list(g.standard_normal(2000) * 2.0 ** g.integers(-140, 128, 2000).astype(np.float64))
    vals = np.array([v for x in vals for v in (x, -x)], dtype=np.float64)
    ours = oracle_mod.f64_to_bf16(vals)
    exact = np.array([_bf16_rne_exact(float(v)) for v in vals], dtype=np.uint16)
    np.testing.assert_array_equal(ours, exact)
    twice = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.count_nonzero(twice != exact) > 100, "the cases do not separate one rounding from two"


def test_tolerance_formula(oracle_mod):
    tol = oracle_mod.gemm_tolerance(np.array([1.0, 1.5, -3.0, 0.0]), np.zeros(4))
    np.testing.assert_array_equal(tol, [2 * 2.0 ** -7, 2 * 2.0 ** -7, 2 * 2.0 ** -6, 2 * 2.0 ** -133])


def test_quant_apply_matches_per_tensor(oracle_mod):
    x = inputs.activations_per_tensor(64)
    bits = inputs.bf16_bits(x)
    q1, s1 = oracle_mod.quant_per_tensor(bits)
    word = int((bits & 0x7FFF).max())
    q2, s2 = oracle_mod.quant_apply(bits, word)
    assert s1 == s2
    np.testing.assert_array_equal(q1, q2)
    q3, s3 = oracle_mod.quant_apply(bits, 0)
    assert s3 == 0
    np.testing.assert_array_equal(q3, np.where(np.signbit(x.float().numpy()), 0x80, 0).astype(np.uint8))


def test_gemm_per_tensor_is_scaled_integer_matmul(oracle_mod):
    """Per-tensor scales: R = s_a * s_b * (A_dec @ B_dec^T), the inner sum exact."""
    qa, _, qb, _ = inputs.gemm_operands(7, 260, 512, seed=21)
    s_a, s_b = np.float32(0.0371), np.float32(0.00917)
    R, T = oracle_mod.gemm_per_tensor(qa, s_a, qb, s_b)
    A = torch.from_numpy(torch_decode(qa))
    B = torch.from_numpy(torch_decode(qb))
    ref = (float(s_a) * float(s_b)) * (A @ B.T).numpy()
    np.testing.assert_allclose(R, ref, rtol=1e-12)
    np.testing.assert_allclose(T, (float(s_a) * float(s_b)) * (A.abs() @ B.abs().T).numpy(), rtol=1e-12)


# ---------------------------------------------------------------- ue8m0
# The ue8m0 reading: scale = smallest power of two 2^e >= amax/448, e clamped
# to [-127, 127], stored as the E8M0 byte e + 127 (255 = NaN).

def _bf16_groups(rows):
    """bf16 bit patterns [len(rows), 128] from float rows (exactly representable)."""
    t = torch.tensor(np.asarray(rows, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_e8m0_exponent_matches_log2(oracle_mod):
    """Every finite bf16 magnitude: byte = clamp(ceil(log2(a/448))) + 127, by the
    math library's log2 (a/448 is never within 1/224 of a power of two from
    above, so float64 log2 decides the ceiling exactly)."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    a = (bits << 16).view(np.float32).astype(np.float64)
    want = np.clip(np.ceil(np.log2(a / 448.0)), -127, 127).astype(np.int64) + 127
    got = np.array([oracle_mod.e8m0_from_amax(float(v)) for v in a])
    assert np.array_equal(got, want)
    assert oracle_mod.e8m0_from_amax(0.0) == 0
    assert oracle_mod.e8m0_from_amax(float("inf")) == 255
    assert oracle_mod.e8m0_from_amax(float("nan")) == 255


def test_ue8m0_worked_values(oracle_mod):
    x = _bf16_groups([[1.0] * 128, [448.0] + [3.0] * 127, [450.0] + [-1.0] * 127])
    q, s = oracle_mod.quant_group128_ue8m0(x)
    assert s[:, 0].tolist() == [119, 127, 128]            # 2^-8, 2^0, 2^1
    dec = oracle_mod.e4m3_decode
    assert set(dec(q[0]).tolist()) == {256.0}               # 1.0 * 2^8
    assert dec(q[1, 0]) == 448.0 and dec(q[1, 1]) == 3.0
    assert dec(q[2, 0]) == 224.0                            # 450/2 = 225 -> 224 (RNE, spacing 16)
    assert dec(q[2, 1]) == -0.5


def test_ue8m0_agrees_with_fp32_path_on_power_of_two_ratios(oracle_mod):
    """When amax/448 is a power of two the fp32 scale is that power of two, so
    both readings give the same codes and the same scale value."""
    g = np.random.default_rng(3)
    rows = []
    for k in range(-20, 21, 5):
        r = g.normal(0, 1, 128) * 448.0 * 2.0 ** k / 6.0
        r = np.clip(r, -0.99 * 448 * 2.0 ** k, 0.99 * 448 * 2.0 ** k)
        r[g.integers(0, 128)] = (448.0 if k % 2 else -448.0) * 2.0 ** k
        rows.append(r)
    x = _bf16_groups(rows)
    q8, s8 = oracle_mod.quant_group128_ue8m0(x)
    q32, s32 = oracle_mod.quant_group128(x)
    assert np.array_equal(q8, q32)
    assert np.array_equal(oracle_mod.e8m0_to_f32(s8), s32)


def test_ue8m0_scale_is_tight_and_codes_round_trip(oracle_mod):
    """amax * 2^-e lies in (224, 448] (the smallest power of two that fits), and
    every code is within half an E4M3 step of x * 2^-e."""
    x = inputs.bf16_bits(inputs.activations_group(64, k=1024))
    q, s = oracle_mod.quant_group128_ue8m0(x)
    xs = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(64, 8, 128)
    e = s.astype(np.int64) - 127
    v = xs * np.ldexp(1.0, -e)[:, :, None]
    am = np.abs(v).max(axis=2)
    assert np.all((am > 224.0) & (am <= 448.0))
    dec = oracle_mod.e4m3_decode(q).reshape(64, 8, 128)
    mag = np.abs(v)
    step = np.where(mag >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(mag, 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(np.abs(dec - v) <= step / 2)


def test_ue8m0_special_groups(oracle_mod):
    tiny = float(np.float32(2.0 ** -133))                  # smallest bf16 subnormal
    x = _bf16_groups([[0.0] * 64 + [-0.0] * 64,
                      [1.0] * 127 + [float("nan")],
                      [2.0] * 127 + [float("-inf")],
                      [tiny] * 128])
    q, s = oracle_mod.quant_group128_ue8m0(x)
    assert s[:, 0].tolist() == [0, 255, 255, 0]
    assert set(q[0, :64].tolist()) == {0x00} and set(q[0, 64:].tolist()) == {0x80}
    assert set(q[1].tolist()) == {0x7F} and set(q[2].tolist()) == {0x7F}
    assert set(q[3].tolist()) == {0x08}                    # 2^-133 * 2^127 = 2^-6, the smallest normal


def test_ue8m0_block128_is_group_rule_on_blocks(oracle_mod):
    """Weight blocks: byte from the block's max |w| (numpy), codes of w * 2^-e."""
    w = inputs.bf16_bits(inputs.weight_tiny())
    q, s = oracle_mod.quant_block128_ue8m0(w)
    n, k = w.shape
    wf = (w.astype(np.uint32) << 16).view(np.float32)
    for nb in range((n + 127) // 128):
        for g in range(k // 128):
            blk = wf[nb * 128:(nb + 1) * 128, g * 128:(g + 1) * 128]
            assert s[nb, g] == oracle_mod.e8m0_from_amax(float(np.abs(blk).max()))
            v = blk.astype(np.float64) * 2.0 ** (127 - int(s[nb, g]))
            want = oracle_mod.e4m3_encode(v.astype(np.float32))
            assert np.array_equal(q[nb * 128:(nb + 1) * 128, g * 128:(g + 1) * 128], want)


def test_gemm_ue8m0_is_integer_matmul_times_powers_of_two(oracle_mod):
    """R = sum_kb 2^(ea+eb) * (A_kb @ B_kb^T), each term exact in float64."""
    qa, _, qb, _ = inputs.gemm_operands(9, 300, 512, seed=33)
    g = np.random.default_rng(34)
    sa = g.integers(100, 150, (9, 4)).astype(np.uint8)
    sb = g.integers(100, 150, (3, 4)).astype(np.uint8)
    R, _ = oracle_mod.gemm_ue8m0(qa, sa, qb, sb)
    A = torch_decode(qa)
    B = torch_decode(qb)
    ref = np.zeros((9, 300))
    for kb in range(4):
        part = A[:, kb * 128:(kb + 1) * 128] @ B[:, kb * 128:(kb + 1) * 128].T
        ea = sa[:, kb].astype(np.int64) - 127
        eb = sb[np.arange(300) // 128, kb].astype(np.int64) - 127
        ref += part * np.ldexp(1.0, ea[:, None] + eb[None, :])
    assert np.array_equal(R, ref)


# ---------------------------------------------------------------- per-channel
def test_per_channel_is_per_tensor_of_each_row(oracle_mod):
    """One scale per row: each row quantised as a one-row tensor."""
    x = inputs.bf16_bits(inputs.activations_per_tensor(40, k=384))
    q, s = oracle_mod.quant_per_channel(x)
    for r in range(40):
        qr, sr = oracle_mod.quant_per_tensor(np.ascontiguousarray(x[r:r + 1]))
        assert np.array_equal(q[r], qr[0]) and np.float32(s[r]) == sr


def test_per_channel_matches_torch(oracle_mod):
    x = inputs.activations_per_tensor(64, k=256)
    xf = x.float()
    amax = xf.abs().amax(dim=1)
    s_ref = (amax / 448.0).numpy()
    q, s = oracle_mod.quant_per_channel(inputs.bf16_bits(x))
    assert np.array_equal(s.view(np.uint32), s_ref.astype(np.float32).view(np.uint32))
    ok = s_ref > 0
    want = torch_encode((xf[ok] / torch.from_numpy(s_ref[ok])[:, None]).numpy())
    assert np.array_equal(q[ok], want)


def test_gemm_per_channel_is_scaled_integer_matmul(oracle_mod):
    qa, _, qb, _ = inputs.gemm_operands(6, 200, 384, seed=41)
    g = np.random.default_rng(42)
    sa = g.uniform(1e-3, 1e-1, 6).astype(np.float32)
    sb = g.uniform(1e-3, 1e-1, 200).astype(np.float32)
    R, T = oracle_mod.gemm_per_channel(qa, sa, qb, sb)
    A = torch_decode(qa)
    B = torch_decode(qb)
    f = sa.astype(np.float64)[:, None] * sb.astype(np.float64)[None, :]
    np.testing.assert_allclose(R, f * (A @ B.T), rtol=1e-12)
    np.testing.assert_allclose(T, f * (np.abs(A) @ np.abs(B).T), rtol=1e-12)
