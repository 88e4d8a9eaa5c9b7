"""ctypes declarations of the fp8q C ABI (include/fp8q.h).

Argument marshalling only: every computation runs in the CUDA library
``libfp8q.so`` built in-tree for sm_100a.  If that library is missing the
load fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_sz = ctypes.c_size_t
_int = ctypes.c_int

# name -> (restype, argtypes); the order follows include/fp8q.h
SIGNATURES = {
    "fp8q_status_string": (ctypes.c_char_p, [_int]),
    "fp8q_abi_version": (_int, []),
    "fp8_act_quant_per_tensor_workspace_size": (_sz, [_i64, _i64]),
    "fp8_act_quant_per_tensor": (_int, [_p, _i64, _i64, _i64, _p, _i64, _p, _p, _sz, _p]),
    "fp8_act_amax_workspace_size": (_sz, [_i64, _i64]),
    "fp8_act_amax": (_int, [_p, _i64, _i64, _i64, _p, _p, _sz, _p]),
    "fp8_act_quant_apply": (_int, [_p, _i64, _i64, _i64, _p, _p, _i64, _p, _p]),
    "fp8_act_quant_group128": (_int, [_p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "fp8_weight_quant_block128": (_int, [_p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "fp8_linear_group128_workspace_size": (_sz, [_i64, _i64, _i64]),
    "fp8_linear_group128": (_int, [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8_act_quant_per_channel": (_int, [_p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "fp8_gemm_per_channel": (_int, [_p, _i64, _p, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8_act_quant_group128_ue8m0": (_int, [_p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "fp8_weight_quant_block128_ue8m0": (_int, [_p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "fp8_block_gemm_workspace_size": (_sz, [_i64, _i64, _i64]),
    "fp8_block_gemm": (_int, [_p, _i64, _p, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8_gemm_per_tensor": (_int, [_p, _i64, _p, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8_block_gemm_ue8m0": (_int, [_p, _i64, _p, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]),
    "fp8_block_gemm_noalloc": (_int, [_p, _i64, _p, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _p]),
    "fp8q_gemm_plan": (_int, [_i64, _i64, _i64, _int, _sz, _p, _p]),
    "fp8q_get_last_device_status": (_int, [_p, _p]),
    "fp8q_device_status": (_int, [_p, _int]),
    "fp8q_set_wait_budget_cycles": (ctypes.c_longlong, [ctypes.c_longlong]),
    "fp8q_launch_count": (ctypes.c_ulonglong, []),
}

NOALLOC_MAX_SCRATCH_BYTES = 8 << 20      # FP8Q_NOALLOC_MAX_SCRATCH_BYTES in include/fp8q.h

STATUS = {
    0: "FP8Q_OK", 1: "FP8Q_ERR_INVALID_ARG", 2: "FP8Q_ERR_UNSUPPORTED_SHAPE",
    3: "FP8Q_ERR_MISALIGNED", 4: "FP8Q_ERR_WORKSPACE", 5: "FP8Q_ERR_CUDA",
    6: "FP8Q_ERR_TIMEOUT", 7: "FP8Q_ERR_NO_DEVICE",
}

_lock = threading.Lock()
_lib = None


class Fp8qError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def load():
    """Load libfp8q.so (raises OSError if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise OSError(f"fp8q CUDA library not built: {LIB_PATH} is missing "
                              "(run __graft_entry__.build())")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def check(status: int, where: str) -> None:
    if status != 0:
        raise Fp8qError(status, where)
