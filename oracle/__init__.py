"""CPU oracle for the FP8 dynamic-quantisation linear path.

TEST INFRASTRUCTURE ONLY.  The test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` call it; the product library never does, and
it shares no code with the CUDA path.  The arithmetic lives in
``fp8q_oracle.c`` (plain C loops, float64 GEMM); this module compiles it with
gcc on first use and marshals numpy arrays into it.

bf16 tensors cross this boundary as ``numpy.uint16`` bit patterns, E4M3 codes
as ``numpy.uint8``.

Every function is pinned by ``tests/test_oracle_pins.py`` against facts that do
not come from the oracle itself (the E4M3 format definition, torch's own
float8 conversion, closed forms, float64 brute force and invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, OpenMP).

    No fast-math and no FMA contraction: every fp32 division and float64 sum
    must round exactly as the C source says.
    """
    if not force and os.path.exists(_LIB_PATH) and (
            os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = ctypes.c_int
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode_bits.argtypes = [_p, _i64, _p]
        lib.oracle_e4m3_encode_range.argtypes = [ctypes.c_uint32, _i64, _p]
        lib.oracle_scale_from_amax.argtypes = [ctypes.c_float]
        lib.oracle_scale_from_amax.restype = ctypes.c_float
        lib.oracle_amax.argtypes = [_p, _i64, _i64, _i64]
        lib.oracle_amax.restype = ctypes.c_float
        lib.oracle_quant_per_tensor.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
        lib.oracle_quant_apply.argtypes = [_p, _i64, _i64, _i64, ctypes.c_uint16, _p, _i64, _p]
        lib.oracle_quant_group128.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
        lib.oracle_quant_block128.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
        lib.oracle_quant_per_channel.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
        lib.oracle_e8m0_from_amax.argtypes = [ctypes.c_float]
        lib.oracle_e8m0_from_amax.restype = ctypes.c_int
        lib.oracle_quant_group128_ue8m0.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
        lib.oracle_quant_block128_ue8m0.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
        lib.oracle_block_gemm.argtypes = [_p, _i64, _p, _p, _i64, _p,
                                          _i64, _i64, _i64, _p, _p]
        lib.oracle_block_gemm_points.argtypes = [_p, _i64, _p, _p, _i64, _p,
                                                 _i64, _p, _p, _i64, _p, _p]
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16_array.argtypes = [_p, _i64, _p]
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _rows(a: np.ndarray, itemsize: int):
    """(rows, cols, row stride in elements) of a 2-D array with unit inner stride."""
    if a.ndim != 2:
        raise ValueError("expected a 2-D array")
    if a.strides[1] != itemsize:
        raise ValueError("inner stride must be 1 element")
    if a.strides[0] % itemsize:
        raise ValueError("row stride must be whole elements")
    return a.shape[0], a.shape[1], a.strides[0] // itemsize


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
    return _load().oracle_set_threads(int(n))


# ---------------------------------------------------------------- codec
def e4m3_decode(codes) -> np.ndarray:
    """float64 value of each E4M3 code (NaN for 0x7F / 0xFF)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    flat_c, flat_o = c.reshape(-1), out.reshape(-1)
    for i in range(flat_c.size):
        flat_o[i] = lib.oracle_e4m3_decode(int(flat_c[i]))
    return out


def e4m3_encode(values) -> np.ndarray:
    """E4M3 code of each fp32 value: round-to-nearest-even, saturate to 448."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32))
    bits = v.view(np.uint32).reshape(-1)
    out = np.empty(bits.size, dtype=np.uint8)
    _load().oracle_e4m3_encode_bits(_ptr(bits), bits.size, _ptr(out))
    return out.reshape(v.shape)


def e4m3_encode_range(first: int, n: int) -> np.ndarray:
    """Codes of the fp32 values whose bit patterns are first, first+1, ..."""
    out = np.empty(int(n), dtype=np.uint8)
    _load().oracle_e4m3_encode_range(ctypes.c_uint32(first), int(n), _ptr(out))
    return out


# ---------------------------------------------------------------- quant
def scale_from_amax(amax: float) -> np.float32:
    return np.float32(_load().oracle_scale_from_amax(float(np.float32(amax))))


def amax(x_bits: np.ndarray) -> np.float32:
    m, k, ld = _rows(x_bits, 2)
    return np.float32(_load().oracle_amax(_ptr(x_bits), m, k, ld))


def quant_per_tensor(x_bits: np.ndarray):
    """(codes [M,K] uint8, scale float32) for a bf16 [M,K] bit array."""
    m, k, ld = _rows(x_bits, 2)
    q = np.empty((m, k), dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    _load().oracle_quant_per_tensor(_ptr(x_bits), m, k, ld, _ptr(q), k, _ptr(s))
    return q, s[0]


def quant_apply(x_bits: np.ndarray, amax_bits: int):
    """(codes, scale) of the apply-only step for a given amax word (the bf16
    bit pattern of the amax; its sign bit is ignored)."""
    m, k, ld = _rows(x_bits, 2)
    q = np.empty((m, k), dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    _load().oracle_quant_apply(_ptr(x_bits), m, k, ld, ctypes.c_uint16(int(amax_bits) & 0xFFFF),
                               _ptr(q), k, _ptr(s))
    return q, s[0]


def quant_per_channel(x_bits: np.ndarray):
    """(codes [M,K] uint8, scales [M] float32): one scale per row."""
    m, k, ld = _rows(x_bits, 2)
    q = np.empty((m, k), dtype=np.uint8)
    s = np.empty(m, dtype=np.float32)
    _load().oracle_quant_per_channel(_ptr(x_bits), m, k, ld, _ptr(q), k, _ptr(s))
    return q, s


def quant_group128(x_bits: np.ndarray):
    """(codes [M,K] uint8, scales [M,K/128] float32)."""
    m, k, ld = _rows(x_bits, 2)
    if k % 128:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((m, k), dtype=np.uint8)
    s = np.empty((m, k // 128), dtype=np.float32)
    _load().oracle_quant_group128(_ptr(x_bits), m, k, ld, _ptr(q), k, _ptr(s))
    return q, s


def quant_block128(w_bits: np.ndarray):
    """(codes [N,K] uint8, scales [ceil(N/128), K/128] float32)."""
    n, k, ld = _rows(w_bits, 2)
    if k % 128:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((n, k), dtype=np.uint8)
    s = np.empty(((n + 127) // 128, k // 128), dtype=np.float32)
    _load().oracle_quant_block128(_ptr(w_bits), n, k, ld, _ptr(q), k, _ptr(s))
    return q, s


# ---------------------------------------------------------------- ue8m0
# [P1] "Benchmarking the Activation Quantization Kernel" names the ue8m0
# scale format (scale_fmt="ue8m0"); the reading of it (smallest power of two
# >= amax/448, E8M0 byte = exponent + 127, 255 = NaN) is in fp8q_oracle.c.
def e8m0_from_amax(amax: float) -> int:
    """E8M0 byte of the power-of-two scale for a group amax."""
    return int(_load().oracle_e8m0_from_amax(float(amax)))


def e8m0_to_f32(b) -> np.ndarray:
    """fp32 values 2^(b-127) of E8M0 bytes (NaN for 255)."""
    b = np.asarray(b, dtype=np.uint8)
    e = np.where(b == 255, 0, b.astype(np.int64) - 127)
    out = np.ldexp(np.ones(b.shape, dtype=np.float64), e).astype(np.float32)
    out[b == 255] = np.nan
    return out


def quant_group128_ue8m0(x_bits: np.ndarray):
    """(codes [M,K] uint8, E8M0 scale bytes [M,K/128] uint8)."""
    m, k, ld = _rows(x_bits, 2)
    if k % 128:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((m, k), dtype=np.uint8)
    s = np.empty((m, k // 128), dtype=np.uint8)
    _load().oracle_quant_group128_ue8m0(_ptr(x_bits), m, k, ld, _ptr(q), k, _ptr(s))
    return q, s


def quant_block128_ue8m0(w_bits: np.ndarray):
    """(codes [N,K] uint8, E8M0 scale bytes [ceil(N/128),K/128] uint8)."""
    n, k, ld = _rows(w_bits, 2)
    if k % 128:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((n, k), dtype=np.uint8)
    s = np.empty(((n + 127) // 128, k // 128), dtype=np.uint8)
    _load().oracle_quant_block128_ue8m0(_ptr(w_bits), n, k, ld, _ptr(q), k, _ptr(s))
    return q, s


# ---------------------------------------------------------------- GEMM
def _gemm_args(qa, sa, qb, sb):
    m, k, lda = _rows(qa, 1)
    n, kb_, ldb = _rows(qb, 1)
    if k != kb_ or k % 128:
        raise ValueError("A and B must share K, a multiple of 128")
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    if sa.shape != (m, k // 128) or sb.shape != ((n + 127) // 128, k // 128):
        raise ValueError("scale shapes must be [M,K/128] and [ceil(N/128),K/128]")
    return m, n, k, lda, ldb, sa, sb


def block_gemm(qa, sa, qb, sb):
    """(R, T): float64 Y = A*B^T with block scales, and the |.|-sum term."""
    m, n, k, lda, ldb, sa, sb = _gemm_args(qa, sa, qb, sb)
    R = np.empty((m, n), dtype=np.float64)
    T = np.empty((m, n), dtype=np.float64)
    _load().oracle_block_gemm(_ptr(qa), lda, _ptr(sa), _ptr(qb), ldb, _ptr(sb),
                              m, n, k, _ptr(R), _ptr(T))
    return R, T


def block_gemm_points(qa, sa, qb, sb, ms, ns):
    """(R, T) of the block GEMM at the points (ms[i], ns[i]) only."""
    m, n, k, lda, ldb, sa, sb = _gemm_args(qa, sa, qb, sb)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    if ms.shape != ns.shape:
        raise ValueError("ms and ns must match")
    if ms.size and (ms.min() < 0 or ms.max() >= m or ns.min() < 0 or ns.max() >= n):
        raise ValueError("point out of range")
    R = np.empty(ms.size, dtype=np.float64)
    T = np.empty(ms.size, dtype=np.float64)
    _load().oracle_block_gemm_points(_ptr(qa), lda, _ptr(sa), _ptr(qb), ldb, _ptr(sb),
                                     k, _ptr(ms), _ptr(ns), ms.size, _ptr(R), _ptr(T))
    return R, T


def gemm_per_tensor(qa, s_a, qb, s_b):
    """(R, T) of the per-tensor-scaled GEMM Y = s_a * s_b * A * B^T ([P2]
    Description and walkthrough: the input is quantised per tensor and the
    projection runs on the codes with the tensor scales): the block GEMM's
    definition with every block scale equal to the tensor scale."""
    m, k = qa.shape
    n = qb.shape[0]
    sa = np.full((m, k // 128), np.float32(s_a), dtype=np.float32)
    sb = np.full(((n + 127) // 128, k // 128), np.float32(s_b), dtype=np.float32)
    return block_gemm(qa, sa, qb, sb)


def gemm_per_channel(qa, sa, qb, sb):
    """(R, T) of the per-channel-scaled GEMM Y[m,n] = sa[m] * sb[n] * sum_k
    A[m,k] B[n,k] (one scale per row of A and per row of B): the block GEMM
    with unit scales gives the exact sums, then one float64 product."""
    m, k = qa.shape
    n = qb.shape[0]
    ones_a = np.ones((m, k // 128), dtype=np.float32)
    ones_b = np.ones(((n + 127) // 128, k // 128), dtype=np.float32)
    R, T = block_gemm(qa, ones_a, qb, ones_b)
    f = np.asarray(sa, np.float64)[:, None] * np.asarray(sb, np.float64)[None, :]
    return R * f, T * np.abs(f)


def gemm_ue8m0(qa, sa_bytes, qb, sb_bytes):
    """(R, T) of the block GEMM with E8M0 scale bytes: the block GEMM's
    definition with each scale 2^(b-127)."""
    return block_gemm(qa, e8m0_to_f32(sa_bytes), qb, e8m0_to_f32(sb_bytes))


def gemm_ue8m0_points(qa, sa_bytes, qb, sb_bytes, ms, ns):
    """gemm_ue8m0 at the listed (m, n) points."""
    return block_gemm_points(qa, e8m0_to_f32(sa_bytes), qb, e8m0_to_f32(sb_bytes), ms, ns)


def f64_to_bf16(values) -> np.ndarray:
    """bf16 bit patterns (uint16) of float64 values, round-to-nearest-even."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float64))
    out = np.empty(v.size, dtype=np.uint16)
    _load().oracle_f64_to_bf16_array(_ptr(v.reshape(-1)), v.size, _ptr(out))
    return out.reshape(v.shape)


def gemm_tolerance(R: np.ndarray, T: np.ndarray) -> np.ndarray:
    """Allowed |Y - R|: 2 bf16 ulps of R plus 1e-3 times the |.|-sum term.

    The ulp is that of bf16 at |R| (2^(floor(log2|R|) - 7), with the
    subnormal floor 2^-133).
    """
    a = np.abs(R)
    e = np.where(a > 0, np.floor(np.log2(np.where(a > 0, a, 1.0))), -126.0)
    e = np.maximum(e, -126.0)
    ulp = np.ldexp(1.0, (e - 7).astype(np.int64))
    return 2.0 * ulp + 1e-3 * T
