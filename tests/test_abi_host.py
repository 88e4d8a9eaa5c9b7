"""Host-side checks of the C ABI: the library loads, exports exactly what
include/fp8q.h declares, and rejects bad arguments with the documented status
before touching a device (these run on machines without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")

OK, INVALID, SHAPE, MISALIGNED, WORKSPACE, CUDA, TIMEOUT, NO_DEVICE = range(8)
A = 0x10000            # fake, 16-byte aligned "device" addresses: never dereferenced
B = 0x20000
C = 0x30000
D = 0x40000


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^(?:const char\*|int|size_t|unsigned long long)\s+(\w+)\s*\(", text, re.M)


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


def test_gemm_argument_checks(cuda_lib):
    f = cuda_lib.fp8_block_gemm
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


def test_no_device_status_without_gpu(cuda_lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    f = cuda_lib.fp8_act_quant_group128
    assert f(A, 4, 128, 128, B, 128, C, None) == NO_DEVICE
    v = ctypes.c_int(0)
    assert cuda_lib.fp8q_device_status(ctypes.byref(v), 0) == NO_DEVICE
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
