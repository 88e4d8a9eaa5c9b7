"""Host-side checks of the C ABI: the library loads, exports exactly what
include/fp8q.h declares, and rejects bad arguments with the documented status
before touching a device (these run on machines without a GPU)."""
import ctypes
import os
import re

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")

OK, INVALID, SHAPE, MISALIGNED, WORKSPACE, CUDA, TIMEOUT, NO_DEVICE = range(8)
A = 0x10000            # fake, 16-byte aligned "device" addresses: never dereferenced
B = 0x20000
C = 0x30000
D = 0x40000


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^(?:const char\*|int|size_t|unsigned long long|long long)\s+(\w+)\s*\(", text, re.M)


def test_header_declares_the_abi():
    names = declared_functions()
    for required in ("fp8_act_quant_per_tensor", "fp8_act_quant_group128", "fp8_block_gemm",
                     "fp8_weight_quant_block128", "fp8q_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(cuda_lib):
    from fp8_dynamic_quantization_b200 import _abi
    for name in declared_functions():
        assert hasattr(cuda_lib, name), name
    assert set(declared_functions()) == set(_abi.SIGNATURES)


def test_status_strings(cuda_lib):
    for code, name in [(0, b"FP8Q_OK"), (2, b"FP8Q_ERR_UNSUPPORTED_SHAPE"), (6, b"FP8Q_ERR_TIMEOUT"),
                       (99, b"FP8Q_ERR_UNKNOWN")]:
        assert cuda_lib.fp8q_status_string(code) == name
    assert cuda_lib.fp8q_abi_version() >> 16 == 1


def test_group128_argument_checks(cuda_lib):
    f = cuda_lib.fp8_act_quant_group128
    assert f(A, 4, 100, 100, B, 100, C, None) == SHAPE           # K % 128
    assert f(A, -1, 128, 128, B, 128, C, None) == INVALID
    assert f(None, 4, 128, 128, B, 128, C, None) == INVALID
    assert f(A, 4, 128, 64, B, 128, C, None) == INVALID           # ldx < K
    assert f(A + 2, 4, 128, 128, B, 128, C, None) == MISALIGNED
    assert f(A, 4, 128, 132, B, 128, C, None) == MISALIGNED      # row pitch 264 B
    assert f(A, 4, 128, 128, B, 128, None, None) == INVALID       # scales
    assert f(A, 0, 128, 128, None, 128, None, None) == OK        # empty: nothing to do


def test_per_tensor_argument_checks(cuda_lib):
    f = cuda_lib.fp8_act_quant_per_tensor
    ws = cuda_lib.fp8_act_quant_per_tensor_workspace_size(64, 2048)
    assert ws >= 8
    assert f(A, 64, 2044, 2048, B, 2048, C, D, ws, None) == SHAPE        # K % 8
    assert f(A, 64, 2048, 2048, B, 2048, None, D, ws, None) == INVALID
    assert f(A, 64, 2048, 2048, B, 2048, C, None, ws, None) == WORKSPACE
    assert f(A, 64, 2048, 2048, B, 2048, C, D, ws - 1, None) == WORKSPACE
    assert f(A, 64, 2048, 2048, B, 2048, C + 1, D, ws, None) == MISALIGNED
    assert f(A, 64, 2048, 2048, B + 4, 2048, C, D, ws, None) == MISALIGNED
    assert f(A, 64, 2048, 2048, B, 2052, C, D, ws, None) == MISALIGNED       # code pitch


def test_amax_apply_argument_checks(cuda_lib):
    ws = cuda_lib.fp8_act_amax_workspace_size(8, 256)
    assert cuda_lib.fp8_act_amax(A, 8, 250, 256, C, D, ws, None) == SHAPE
    assert cuda_lib.fp8_act_amax(A, 8, 256, 256, None, D, ws, None) == INVALID
    assert cuda_lib.fp8_act_amax(A, 8, 256, 256, C, D, 0, None) == WORKSPACE
    assert cuda_lib.fp8_act_quant_apply(A, 8, 256, 256, None, B, 256, C, None) == INVALID
    assert cuda_lib.fp8_act_quant_apply(A, 8, 256, 256, C + 2, B, 256, C, None) == MISALIGNED


def test_block128_argument_checks(cuda_lib):
    f = cuda_lib.fp8_weight_quant_block128
    assert f(A, 200, 192, 192, B, 192, C, None) == SHAPE
    assert f(A, 200, 256, 256, B, 256, None, None) == INVALID
    assert f(A, 200, 256, 256, B + 4, 256, C, None) == MISALIGNED


def _gemm_entry(cuda_lib, name):
    """fp8_block_gemm, or fp8_block_gemm_noalloc behind the same argument
    list (its workspace arguments dropped)."""
    if name == "fp8_block_gemm":
        return cuda_lib.fp8_block_gemm
    g = cuda_lib.fp8_block_gemm_noalloc
    return lambda qa, lda, sa, qb, ldb, sb, y, ldy, m, n, k, ws, wsb, st: g(qa, lda, sa, qb, ldb, sb, y, ldy,
                                                                           m, n, k, st)


@pytest.mark.parametrize("name", ["fp8_block_gemm", "fp8_block_gemm_noalloc"])
def test_gemm_argument_checks(cuda_lib, name):
    """Both GEMM entry points report argument errors with the same codes,
    before they look for a device (this host has none) or plan a launch."""
    f = _gemm_entry(cuda_lib, name)
    assert f(A, 200, B, C, 200, D, A, 64, 16, 64, 200, None, 0, None) == SHAPE     # K % 128
    assert f(A, 256, B, C, 256, D, A, 64, -1, 64, 256, None, 0, None) == INVALID
    assert f(A, 256, B, C, 256, D, A, 64, 0, 64, 256, None, 0, None) == OK          # empty M
    assert f(A, 256, B, C, 256, D, A, 64, 16, 0, 256, None, 0, None) == OK          # empty N
    assert f(None, 256, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == INVALID
    assert f(A, 128, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == INVALID    # lda < K
    assert f(A, 256, B, C, 256, D, A, 32, 16, 64, 256, None, 0, None) == INVALID    # ldy < N
    assert f(A + 16 * 0 + 8, 256, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == MISALIGNED
    assert f(A, 264, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == MISALIGNED  # lda pitch
    assert f(A, 256, B, C, 256, D, A, 60, 16, 60, 256, None, 0, None) == MISALIGNED  # ldy pitch
    assert f(A, 256, B + 1, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == MISALIGNED
    # a skinny shape beyond the no-alloc scratch (32 x 32776 x 8320) with a
    # null output: the pointer error wins over any workspace question
    assert f(A, 8320, B, C, 8320, D, None, 32776, 32, 32776, 8320, None, 0, None) == INVALID
    # sizes beyond INT_MAX: unsupported, before any launch plan is made
    big = 1 << 31
    assert f(A, 256, B, C, 256, D, A, big, 16, big, 256, None, 0, None) == SHAPE
    assert f(A, 256, B, C, 256, D, A, 64, big, 64, 256, None, 0, None) == SHAPE
    assert f(A, big * 128, B, C, big * 128, D, A, 64, 16, 64, big * 128, None, 0, None) == SHAPE


def test_no_device_status_without_gpu(cuda_lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    f = cuda_lib.fp8_act_quant_group128
    assert f(A, 4, 128, 128, B, 128, C, None) == NO_DEVICE
    v = ctypes.c_int(0)
    assert cuda_lib.fp8q_device_status(ctypes.byref(v), 0) == NO_DEVICE
    assert cuda_lib.fp8q_get_last_device_status(None, ctypes.byref(v)) == NO_DEVICE
    assert cuda_lib.fp8q_get_last_device_status(None, None) == INVALID
    # valid arguments: the no-alloc GEMM gets as far as looking for a device
    assert cuda_lib.fp8_block_gemm_noalloc(A, 256, B, C, 256, D, A, 64, 16, 64, 256, None) == NO_DEVICE
    assert cuda_lib.fp8_block_gemm_workspace_size(16, 64, 256) == 0


def test_python_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from fp8_dynamic_quantization_b200 import _abi
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(OSError):
        _abi.load()


@pytest.mark.parametrize("name", ["fp8_gemm_per_tensor", "fp8_gemm_per_channel", "fp8_block_gemm_ue8m0"])
def test_scaled_gemm_variants_argument_checks(cuda_lib, name):
    """The per-tensor, per-channel and ue8m0 GEMMs validate like fp8_block_gemm;
    only the ue8m0 one accepts byte-aligned scale pointers."""
    f = getattr(cuda_lib, name)
    assert f(A, 200, B, C, 200, D, A, 64, 16, 64, 200, None, 0, None) == SHAPE     # K % 128
    assert f(A, 256, B, C, 256, D, A, 64, 0, 64, 256, None, 0, None) == OK          # empty M
    assert f(None, 256, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == INVALID
    assert f(A, 256, None, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == INVALID
    assert f(A, 128, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == INVALID    # lda < K
    assert f(A, 264, B, C, 256, D, A, 64, 16, 64, 256, None, 0, None) == MISALIGNED  # lda pitch
    odd_scales = f(A, 256, B + 1, C, 256, D + 1, A, 64, 16, 64, 256, None, 0, None)
    if name == "fp8_block_gemm_ue8m0":
        assert odd_scales != MISALIGNED
    else:
        assert odd_scales == MISALIGNED


def test_linear_group128_argument_checks(cuda_lib):
    f = cuda_lib.fp8_linear_group128
    assert f(A, 200, C, 200, D, B, 64, 16, 64, 200, None, 0, None) == SHAPE        # K % 128
    assert f(A, 256, C, 256, D, B, 64, 0, 64, 256, None, 0, None) == OK            # empty M
    assert f(A, 256, C, 256, D, B, 64, -1, 64, 256, None, 0, None) == INVALID


@pytest.mark.parametrize("name", ["fp8_act_quant_per_channel", "fp8_act_quant_group128_ue8m0"])
def test_new_quant_argument_checks(cuda_lib, name):
    f = getattr(cuda_lib, name)
    assert f(A, 4, 130, 130, B, 136, C, None) == SHAPE                             # K % 8 / % 128
    assert f(A, 4, 256, 256, B, 256, None, None) == INVALID
    assert f(A + 8, 4, 256, 256, B, 256, C, None) == MISALIGNED
    assert f(A, 0, 256, 256, B, 256, C, None) == OK                                # empty


# ------------------------------------------------------------ launch plans
PLAN_KEYS = ("swap", "pair", "bn", "stages", "splits", "tiles_p", "tiles_q", "units", "grid",
             "tail_tiles", "tail_splits")
NO_CAP = (1 << 64) - 1
NOALLOC_CAP = 8 << 20


def gemm_plan(lib, m, n, k, sms=148, cap=NO_CAP):
    out = (ctypes.c_int * 11)()
    ws = ctypes.c_size_t(0)
    rc = lib.fp8q_gemm_plan(m, n, k, sms, cap, out, ctypes.byref(ws))
    assert rc == OK
    plan = dict(zip(PLAN_KEYS, list(out)))
    plan["ws"] = ws.value
    return plan


def test_plan_argument_checks(cuda_lib):
    out = (ctypes.c_int * 11)()
    ws = ctypes.c_size_t(0)
    assert cuda_lib.fp8q_gemm_plan(4, 4, 100, 148, NO_CAP, out, ctypes.byref(ws)) == SHAPE
    assert cuda_lib.fp8q_gemm_plan(0, 4, 128, 148, NO_CAP, out, ctypes.byref(ws)) == INVALID
    assert cuda_lib.fp8q_gemm_plan(4, 4, 128, 0, NO_CAP, out, ctypes.byref(ws)) == INVALID
    assert cuda_lib.fp8q_gemm_plan(4, 4, 128, 148, NO_CAP, None, ctypes.byref(ws)) == INVALID


def test_plan_prefill_tiles_and_split_last_wave(cuda_lib):
    # 4096 x 7168: CTA pairs, 16 x 28 = 448 tiles of 256 x 256 = 6 waves of
    # 74 pairs + 4; the 4 are split into min(74 // 4, 56 // 2) = 18 K ranges
    p = gemm_plan(cuda_lib, 4096, 7168, 7168)
    assert (p["swap"], p["pair"], p["bn"], p["splits"]) == (0, 1, 256, 1)
    assert (p["tiles_p"], p["tiles_q"], p["tail_tiles"], p["tail_splits"]) == (16, 28, 4, 18)
    assert p["units"] == 444 + 4 * 18 and p["grid"] == 148
    assert p["ws"] == 4 * 18 * 256 * 256 * 4
    # last waves of 42 and 56 tiles hold more than half the pairs: whole tiles
    for n, tail in ((18432, 42), (24576, 56)):
        p = gemm_plan(cuda_lib, 4096, n, 7168)
        assert p["pair"] == 1 and (p["tiles_p"] * p["tiles_q"]) % 74 == tail
        assert (p["tail_tiles"], p["units"], p["ws"]) == (0, p["tiles_p"] * p["tiles_q"], 0)


def test_plan_tile_choice_by_m_and_n(cuda_lib):
    def key(m, n):
        p = gemm_plan(cuda_lib, m, n, 7168)
        return ("swap" if p["swap"] else "pair" if p["pair"] else "normal", p["bn"])
    assert key(1, 18432) == ("swap", 16) and key(16, 7168) == ("swap", 16)
    assert key(17, 2048) == ("swap", 32) and key(32, 18432) == ("swap", 32)
    for m in (33, 64, 128):
        assert key(m, 2048) == ("normal", 128)
        assert key(m, 7168) == ("normal", 256)
        assert key(m, 18432) == ("normal", 128)
    for m in (129, 256, 512):
        for n in (2048, 7168, 16384):
            assert key(m, n) == ("normal", 256)
        for n in (16385, 18432, 24576):
            assert key(m, n) == ("pair", 256)
    for m in (513, 1024, 4096):
        for n in (2048, 7168, 18432):
            assert key(m, n) == ("pair", 256)


def test_plan_split_k_fills_the_sms_and_respects_a_cap(cuda_lib):
    # 64 x 7168: 1 x 28 tiles of 128 x 256 -> 148 // 28 = 5 K ranges
    p = gemm_plan(cuda_lib, 64, 7168, 7168)
    assert (p["splits"], p["units"]) == (5, 28 * 5)
    assert p["ws"] == 5 * 64 * 7168 * 4
    # with the no-alloc scratch as the cap: 8 MiB // (64 * 7168 * 4) = 4
    q = gemm_plan(cuda_lib, 64, 7168, 7168, cap=NOALLOC_CAP)
    assert (q["splits"], q["units"]) == (4, 28 * 4) and q["ws"] <= NOALLOC_CAP
    # skinny M: 144 swapped weight tiles, too few K blocks to split further
    p = gemm_plan(cuda_lib, 16, 18432, 7168)
    assert (p["swap"], p["tiles_p"], p["tiles_q"], p["splits"], p["ws"]) == (1, 144, 1, 1, 0)


def test_plan_cap_cuts_the_split_tail_and_the_swapped_minimum(cuda_lib):
    # 4000 x 7100 x 4608: 448 pair tiles, tail of 4, 36 K blocks -> 18 ranges,
    # 18 MiB of partials; under the 8 MiB cap (1 MiB per range) 8 ranges
    p = gemm_plan(cuda_lib, 4000, 7100, 4608)
    assert (p["tail_tiles"], p["tail_splits"]) == (4, 18) and p["ws"] > NOALLOC_CAP
    q = gemm_plan(cuda_lib, 4000, 7100, 4608, cap=NOALLOC_CAP)
    assert (q["tail_tiles"], q["tail_splits"]) == (4, 8) and q["ws"] <= NOALLOC_CAP
    # single-CTA tiles (M <= 512): 512 x 7100 x 4608 -> 4 x 28 = 112 tiles, one
    # wave, nothing to split
    p = gemm_plan(cuda_lib, 512, 7100, 4608)
    assert (p["pair"], p["tail_tiles"], p["units"]) == (0, 0, 112)
    # 32 swapped tokens with 65 K blocks need 2 K ranges whatever the cap
    q = gemm_plan(cuda_lib, 32, 32776, 8320, cap=NOALLOC_CAP)
    assert q["swap"] == 1 and q["splits"] == 2 and q["ws"] == 2 * 32 * 32776 * 4 > NOALLOC_CAP


def test_plan_depends_on_the_sm_count(cuda_lib):
    # 4096 x 7168 on 132 SMs (66 pairs): 448 = 6 * 66 + 52 -> more than half a wave
    p = gemm_plan(cuda_lib, 4096, 7168, 7168, sms=132)
    assert (p["tail_tiles"], p["grid"]) == (0, 132)


@settings(max_examples=400, deadline=None)
@given(m=st.one_of(st.integers(1, 40), st.integers(1, 600), st.integers(1, 20000)),
       n=st.one_of(st.integers(1, 2100), st.integers(1, 40000)), g=st.integers(1, 128),
       sms=st.integers(4, 80).map(lambda h: 2 * h), capped=st.booleans())
def test_plan_invariants(cuda_lib, m, n, g, sms, capped):
    """Whatever the shape, SM count and workspace cap: the tiles cover the
    output, every work unit has at least one K block, the grid fits the SMs
    (an even count for CTA pairs), and the workspace is what the partials
    need (within the cap unless the swapped minimum of two K ranges is
    forced)."""
    k = 128 * g
    cap = NOALLOC_CAP if capped else NO_CAP
    p = gemm_plan(cuda_lib, m, n, k, sms=sms, cap=cap)
    rows = 256 if p["pair"] else 128
    if p["swap"]:
        assert not p["pair"] and p["bn"] <= 128
        assert p["tiles_p"] == -(-n // 128) and p["tiles_q"] == -(-m // p["bn"])
    else:
        assert p["tiles_p"] == -(-m // rows) and p["tiles_q"] == -(-n // p["bn"])
    tiles = p["tiles_p"] * p["tiles_q"]
    assert 1 <= p["splits"] <= g
    if p["tail_tiles"]:
        slots = sms // 2 if p["pair"] else sms
        assert p["splits"] == 1 and not p["swap"]
        assert tiles > slots and p["tail_tiles"] == tiles % slots
        assert 2 <= p["tail_splits"] <= min(slots // p["tail_tiles"], g // 2)
        assert p["units"] == tiles - p["tail_tiles"] + p["tail_tiles"] * p["tail_splits"]
        assert p["ws"] == p["tail_tiles"] * p["tail_splits"] * rows * p["bn"] * 4
    else:
        assert p["tail_splits"] == 1 and p["units"] == tiles * p["splits"]
        ldw = -(-n // 8) * 8
        assert p["ws"] == (p["splits"] * m * ldw * 4 if p["splits"] > 1 else 0)
    if p["pair"]:
        assert p["grid"] % 2 == 0 and p["grid"] == 2 * max(1, min(p["units"], sms // 2))
    else:
        assert p["grid"] == max(1, min(p["units"], sms))
    # the swapped kernel takes at most 64 K blocks per unit, cap or not
    forced = p["swap"] and g > 64 and p["splits"] == -(-g // 64)
    assert p["ws"] <= cap or forced
