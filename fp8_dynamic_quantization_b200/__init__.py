"""fp8q: the FP8 (E4M3) dynamic-quantisation linear path on NVIDIA B200.

Thin PyTorch binding over the C ABI in ``include/fp8q.h``.  PyTorch provides
device memory and streams; every step of the path runs in the library's own
sm_100a kernels (``libfp8q.so``, built in-tree).  There is no CPU fallback:
calls raise if the library is missing or the device is not sm_100.

    q, s   = act_quant_per_tensor(x)      # exact amax, s = amax/448, codes
    q, S   = act_quant_group128(x)        # one scale per 1x128 group along K
    qb, sb = weight_quant_block128(w)     # one scale per 128x128 block
    y      = block_gemm(q, S, qb, sb)     # bf16 Y = A * B^T, block-scaled
    y      = linear(x, qb, sb)            # group quant + block GEMM
    y      = gemm_per_tensor(q, s, qw, sw)  # per-tensor scales: Y = s*sw*A*B^T

Codes are returned as ``torch.float8_e4m3fn`` tensors, scales as float32.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi

__all__ = [
    "act_quant_per_tensor", "act_amax", "act_quant_apply", "act_quant_group128",
    "weight_quant_block128", "act_quant_group128_ue8m0", "weight_quant_block128_ue8m0",
    "block_gemm_ue8m0", "linear_ue8m0", "act_quant_per_channel", "gemm_per_channel",
    "linear_per_channel",
    "block_gemm", "linear", "linear_fused", "gemm_per_tensor", "linear_per_tensor",
    "device_status", "stream_status",
    "per_tensor_sharded", "Fp8qError", "library",
]

Fp8qError = _abi.Fp8qError
E4M3 = torch.float8_e4m3fn

_workspaces: dict = {}


def library():
    """The loaded ctypes handle of libfp8q.so."""
    return _abi.load()


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _rows(t: torch.Tensor, name: str):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.size(1) > 1 and t.stride(1) != 1:
        raise ValueError(f"{name} must have unit inner stride")
    return t.size(0), t.size(1), max(t.stride(0), t.size(1))


def _workspace(kind: str, dev: torch.device, nbytes: int, zero: bool) -> torch.Tensor:
    """A cached device workspace per (kind, device, stream), grown on demand.
    Zero-filled ones are filled once at allocation; the kernels leave them
    ready for the next call on the same stream."""
    key = (kind, dev.index, _stream(dev))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = (torch.zeros if zero else torch.empty)(max(nbytes, 16), dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


def act_quant_per_tensor(x: torch.Tensor):
    """Per-tensor dynamic quantisation of bf16 x[M,K] (K % 8 == 0).

    Returns (codes [M,K] float8_e4m3fn, scale [1] float32) with
    scale = fl32(max|x| / 448) and codes = e4m3_rne_sat(fl32(x / scale)).
    """
    lib = _abi.load()
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    M, K, ldx = _rows(x, "x")
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty(1, dtype=torch.float32, device=x.device)
    nbytes = lib.fp8_act_quant_per_tensor_workspace_size(M, K)
    ws = _workspace("per_tensor", x.device, nbytes, zero=False)
    _abi.check(lib.fp8_act_quant_per_tensor(x.data_ptr(), M, K, ldx, q.data_ptr(), K, s.data_ptr(),
                                            ws.data_ptr(), ws.numel(), _stream(x.device)),
               "fp8_act_quant_per_tensor")
    return q.view(E4M3), s


def act_amax(x: torch.Tensor) -> torch.Tensor:
    """bf16 bit pattern of max|x| as an int32 [1] tensor (0..0x7FFF for
    finite and Inf values, larger for NaN); the max of several such words is
    the amax of the union of the inputs."""
    lib = _abi.load()
    M, K, ldx = _rows(x, "x")
    out = torch.empty(1, dtype=torch.int32, device=x.device)
    nbytes = lib.fp8_act_amax_workspace_size(M, K)
    ws = _workspace("amax", x.device, nbytes, zero=False)
    _abi.check(lib.fp8_act_amax(x.data_ptr(), M, K, ldx, out.data_ptr(), ws.data_ptr(), ws.numel(),
                                _stream(x.device)), "fp8_act_amax")
    return out


def act_quant_apply(x: torch.Tensor, amax_bits: torch.Tensor):
    """Codes and scale of bf16 x[M,K] for a given amax word (see act_amax)."""
    lib = _abi.load()
    M, K, ldx = _rows(x, "x")
    if amax_bits.dtype != torch.int32 or amax_bits.numel() != 1 or amax_bits.device != x.device:
        raise ValueError("amax_bits must be an int32 [1] tensor on x's device")
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty(1, dtype=torch.float32, device=x.device)
    _abi.check(lib.fp8_act_quant_apply(x.data_ptr(), M, K, ldx, amax_bits.data_ptr(), q.data_ptr(), K,
                                       s.data_ptr(), _stream(x.device)), "fp8_act_quant_apply")
    return q.view(E4M3), s


def act_quant_group128(x: torch.Tensor):
    """Per-1x128-group quantisation of bf16 x[M,K] (K % 128 == 0).

    Returns (codes [M,K] float8_e4m3fn, scales [M,K/128] float32)."""
    lib = _abi.load()
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    M, K, ldx = _rows(x, "x")
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _abi.check(lib.fp8_act_quant_group128(x.data_ptr(), M, K, ldx, q.data_ptr(), K, s.data_ptr(),
                                          _stream(x.device)), "fp8_act_quant_group128")
    return q.view(E4M3), s


def weight_quant_block128(w: torch.Tensor):
    """Per-128x128-block quantisation of a bf16 weight w[N,K].

    Returns (codes [N,K] float8_e4m3fn, scales [ceil(N/128), K/128] float32)."""
    lib = _abi.load()
    if w.dtype != torch.bfloat16:
        raise TypeError("w must be bfloat16")
    N, K, ldw = _rows(w, "w")
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    s = torch.empty(((N + 127) // 128, K // 128), dtype=torch.float32, device=w.device)
    _abi.check(lib.fp8_weight_quant_block128(w.data_ptr(), N, K, ldw, q.data_ptr(), K, s.data_ptr(),
                                             _stream(w.device)), "fp8_weight_quant_block128")
    return q.view(E4M3), s


def act_quant_per_channel(x: torch.Tensor):
    """Per-channel (per-row) quantisation of bf16 x[M,K] (K % 8 == 0).

    Returns (codes [M,K] float8_e4m3fn, scales [M] float32)."""
    lib = _abi.load()
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    M, K, ldx = _rows(x, "x")
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty(M, dtype=torch.float32, device=x.device)
    _abi.check(lib.fp8_act_quant_per_channel(x.data_ptr(), M, K, ldx, q.data_ptr(), K, s.data_ptr(),
                                             _stream(x.device)), "fp8_act_quant_per_channel")
    return q.view(E4M3), s


def act_quant_group128_ue8m0(x: torch.Tensor):
    """Per-1x128-group quantisation with power-of-two (ue8m0) scales.

    Returns (codes [M,K] float8_e4m3fn, E8M0 scale bytes [M,K/128] uint8;
    scale value 2^(b-127), 255 = NaN)."""
    lib = _abi.load()
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    M, K, ldx = _rows(x, "x")
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.uint8, device=x.device)
    _abi.check(lib.fp8_act_quant_group128_ue8m0(x.data_ptr(), M, K, ldx, q.data_ptr(), K, s.data_ptr(),
                                                _stream(x.device)), "fp8_act_quant_group128_ue8m0")
    return q.view(E4M3), s


def weight_quant_block128_ue8m0(w: torch.Tensor):
    """Per-128x128-block quantisation with power-of-two (ue8m0) scales.

    Returns (codes [N,K] float8_e4m3fn, E8M0 bytes [ceil(N/128), K/128] uint8)."""
    lib = _abi.load()
    if w.dtype != torch.bfloat16:
        raise TypeError("w must be bfloat16")
    N, K, ldw = _rows(w, "w")
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    s = torch.empty(((N + 127) // 128, K // 128), dtype=torch.uint8, device=w.device)
    _abi.check(lib.fp8_weight_quant_block128_ue8m0(w.data_ptr(), N, K, ldw, q.data_ptr(), K, s.data_ptr(),
                                                   _stream(w.device)), "fp8_weight_quant_block128_ue8m0")
    return q.view(E4M3), s


def _codes(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype not in (E4M3, torch.uint8):
        raise TypeError(f"{name} must be float8_e4m3fn or uint8 codes")
    return t


def block_gemm(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
               out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 Y[M,N] = A * B^T with A scaled per 1x128 group (sa [M,K/128]) and
    B per 128x128 block (sb [ceil(N/128),K/128]); fp32 accumulation."""
    lib = _abi.load()
    M, K, lda = _rows(_codes(qa, "qa"), "qa")
    N, Kb, ldb = _rows(_codes(qb, "qb"), "qb")
    if K != Kb:
        raise ValueError("qa and qb must share K")
    G = K // 128
    for t, shape, name in ((sa, (M, G), "sa"), (sb, ((N + 127) // 128, G), "sb")):
        if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 tensor of shape {shape}")
    if out is None:
        # the output row pitch must be a multiple of 16 bytes: pad odd N
        ldy_alloc = (N + 7) // 8 * 8
        out = torch.empty((M, ldy_alloc), dtype=torch.bfloat16, device=qa.device)[:, :N]
    _, _, ldy = _rows(out, "out")
    nbytes = lib.fp8_block_gemm_workspace_size(M, N, K)
    ws_ptr, ws_len = None, 0
    if nbytes:
        ws = _workspace("gemm", qa.device, nbytes, zero=False)
        ws_ptr, ws_len = ws.data_ptr(), ws.numel()
    _abi.check(lib.fp8_block_gemm(qa.data_ptr(), lda, sa.data_ptr(), qb.data_ptr(), ldb, sb.data_ptr(),
                                  out.data_ptr(), ldy, M, N, K, ws_ptr, ws_len, _stream(qa.device)),
               "fp8_block_gemm")
    return out


def gemm_per_tensor(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 Y[M,N] = sa * sb * A * B^T with one fp32 scale per operand
    (sa, sb: float32 [1] device tensors, e.g. from act_quant_per_tensor)."""
    lib = _abi.load()
    M, K, lda = _rows(_codes(qa, "qa"), "qa")
    N, Kb, ldb = _rows(_codes(qb, "qb"), "qb")
    if K != Kb:
        raise ValueError("qa and qb must share K")
    for t, name in ((sa, "sa"), (sb, "sb")):
        if t.dtype != torch.float32 or t.numel() != 1 or not t.is_cuda:
            raise ValueError(f"{name} must be a float32 [1] CUDA tensor")
    if out is None:
        ldy_alloc = (N + 7) // 8 * 8
        out = torch.empty((M, ldy_alloc), dtype=torch.bfloat16, device=qa.device)[:, :N]
    _, _, ldy = _rows(out, "out")
    nbytes = lib.fp8_block_gemm_workspace_size(M, N, K)
    ws_ptr, ws_len = None, 0
    if nbytes:
        ws = _workspace("gemm", qa.device, nbytes, zero=False)
        ws_ptr, ws_len = ws.data_ptr(), ws.numel()
    _abi.check(lib.fp8_gemm_per_tensor(qa.data_ptr(), lda, sa.data_ptr(), qb.data_ptr(), ldb, sb.data_ptr(),
                                       out.data_ptr(), ldy, M, N, K, ws_ptr, ws_len, _stream(qa.device)),
               "fp8_gemm_per_tensor")
    return out


def linear_per_tensor(x: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor) -> torch.Tensor:
    """The dynamic per-tensor FP8 linear method: per-tensor quantisation of x
    (exact amax, scale = amax/448), then the per-tensor-scaled GEMM against
    weight codes qb with scale sb."""
    qa, sa = act_quant_per_tensor(x)
    return gemm_per_tensor(qa, sa, qb, sb)


def gemm_per_channel(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 Y[M,N] = sa[m] * sb[n] * A * B^T with one fp32 scale per row of A
    (sa [M]) and per row of B (sb [N], an output channel)."""
    lib = _abi.load()
    M, K, lda = _rows(_codes(qa, "qa"), "qa")
    N, Kb, ldb = _rows(_codes(qb, "qb"), "qb")
    if K != Kb:
        raise ValueError("qa and qb must share K")
    if sa.dtype != torch.float32 or tuple(sa.shape) != (M,) or not sa.is_contiguous():
        raise ValueError("sa must be a contiguous float32 [M] tensor")
    if sb.dtype != torch.float32 or tuple(sb.shape) != (N,) or not sb.is_contiguous():
        raise ValueError("sb must be a contiguous float32 [N] tensor")
    if out is None:
        ldy_alloc = (N + 7) // 8 * 8
        out = torch.empty((M, ldy_alloc), dtype=torch.bfloat16, device=qa.device)[:, :N]
    _, _, ldy = _rows(out, "out")
    nbytes = lib.fp8_block_gemm_workspace_size(M, N, K)
    ws_ptr, ws_len = None, 0
    if nbytes:
        ws = _workspace("gemm", qa.device, nbytes, zero=False)
        ws_ptr, ws_len = ws.data_ptr(), ws.numel()
    _abi.check(lib.fp8_gemm_per_channel(qa.data_ptr(), lda, sa.data_ptr(), qb.data_ptr(), ldb, sb.data_ptr(),
                                        out.data_ptr(), ldy, M, N, K, ws_ptr, ws_len, _stream(qa.device)),
               "fp8_gemm_per_channel")
    return out


def linear_per_channel(x: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor) -> torch.Tensor:
    """The dynamic FP8 linear method with per-channel scales: per-token
    quantisation of x, then the GEMM against weight codes qb with one scale
    per output channel (sb [N])."""
    qa, sa = act_quant_per_channel(x)
    return gemm_per_channel(qa, sa, qb, sb)


def block_gemm_ue8m0(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 Y[M,N] = A * B^T with E8M0 (power-of-two) block scales, applied
    by the tensor cores: sa uint8 [M,K/128], sb uint8 [ceil(N/128),K/128]."""
    lib = _abi.load()
    M, K, lda = _rows(_codes(qa, "qa"), "qa")
    N, Kb, ldb = _rows(_codes(qb, "qb"), "qb")
    if K != Kb:
        raise ValueError("qa and qb must share K")
    if sa.dtype != torch.uint8 or tuple(sa.shape) != (M, K // 128) or not sa.is_contiguous():
        raise ValueError("sa must be a contiguous uint8 [M, K/128] tensor")
    if sb.dtype != torch.uint8 or tuple(sb.shape) != ((N + 127) // 128, K // 128) or not sb.is_contiguous():
        raise ValueError("sb must be a contiguous uint8 [ceil(N/128), K/128] tensor")
    if out is None:
        ldy_alloc = (N + 7) // 8 * 8
        out = torch.empty((M, ldy_alloc), dtype=torch.bfloat16, device=qa.device)[:, :N]
    _, _, ldy = _rows(out, "out")
    nbytes = lib.fp8_block_gemm_workspace_size(M, N, K)
    ws_ptr, ws_len = None, 0
    if nbytes:
        ws = _workspace("gemm", qa.device, nbytes, zero=False)
        ws_ptr, ws_len = ws.data_ptr(), ws.numel()
    _abi.check(lib.fp8_block_gemm_ue8m0(qa.data_ptr(), lda, sa.data_ptr(), qb.data_ptr(), ldb, sb.data_ptr(),
                                        out.data_ptr(), ldy, M, N, K, ws_ptr, ws_len, _stream(qa.device)),
               "fp8_block_gemm_ue8m0")
    return out


def linear_ue8m0(x: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor) -> torch.Tensor:
    """The dynamic FP8 linear method with ue8m0 scales: group-128 quantise x
    with power-of-two scales, then the block-scaled GEMM against weight codes
    qb with E8M0 block scales sb."""
    qa, sa = act_quant_group128_ue8m0(x)
    return block_gemm_ue8m0(qa, sa, qb, sb)


def linear_fused(x: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """linear() in one call, bit-identical to act_quant_group128 followed by
    block_gemm: the GEMM is launched as a programmatic dependent of the
    quantisation, so its weight loads start while the tokens are quantised."""
    lib = _abi.load()
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    M, K, ldx = _rows(x, "x")
    N, Kb, ldb = _rows(_codes(qb, "qb"), "qb")
    if K != Kb:
        raise ValueError("x and qb must share K")
    if sb.dtype != torch.float32 or tuple(sb.shape) != ((N + 127) // 128, K // 128) or not sb.is_contiguous():
        raise ValueError("sb must be a contiguous float32 [ceil(N/128), K/128] tensor")
    if out is None:
        ldy_alloc = (N + 7) // 8 * 8
        out = torch.empty((M, ldy_alloc), dtype=torch.bfloat16, device=x.device)[:, :N]
    _, _, ldy = _rows(out, "out")
    nbytes = lib.fp8_linear_group128_workspace_size(M, N, K)
    ws_ptr, ws_len = None, 0
    if nbytes:
        ws = _workspace("linear", x.device, nbytes, zero=False)
        ws_ptr, ws_len = ws.data_ptr(), ws.numel()
    _abi.check(lib.fp8_linear_group128(x.data_ptr(), ldx, qb.data_ptr(), ldb, sb.data_ptr(), out.data_ptr(), ldy,
                                       M, N, K, ws_ptr, ws_len, _stream(x.device)), "fp8_linear_group128")
    return out


def linear(x: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor) -> torch.Tensor:
    """The dynamic FP8 linear method: group-128 quantise x, then the block
    GEMM against pre-quantised weight codes qb with block scales sb."""
    qa, sa = act_quant_group128(x)
    return block_gemm(qa, sa, qb, sb)


def device_status(reset: bool = True) -> int:
    """Synchronise the device and return the first device-side error
    recorded by a kernel on any stream (0 = none; 6 = a bounded wait timed
    out)."""
    lib = _abi.load()
    v = ctypes.c_int(0)
    _abi.check(lib.fp8q_device_status(ctypes.byref(v), int(reset)), "fp8q_device_status")
    return v.value


def stream_status(stream: torch.cuda.Stream | None = None) -> int:
    """Wait for `stream` (default: the current stream) only, then return and
    clear the first device-side error its kernels recorded (0 = none)."""
    lib = _abi.load()
    st = stream if stream is not None else torch.cuda.current_stream()
    v = ctypes.c_int(0)
    _abi.check(lib.fp8q_get_last_device_status(st.cuda_stream, ctypes.byref(v)), "fp8q_get_last_device_status")
    return v.value


def per_tensor_sharded(x: torch.Tensor, group=None, amax_fn=None, apply_fn=None):
    """Per-tensor quantisation of a tensor whose rows are sharded across the
    ranks of a torch.distributed process group: local amax word, one 4-byte
    MAX all-reduce, then the local apply.  Exact: max is order-free.

    amax_fn(x) -> int32 [1] tensor and apply_fn(x, amax_bits) -> (q, s)
    default to the CUDA entry points act_amax / act_quant_apply."""
    import torch.distributed as dist
    amax_fn = amax_fn or act_amax
    apply_fn = apply_fn or act_quant_apply
    word = amax_fn(x)
    dist.all_reduce(word, op=dist.ReduceOp.MAX, group=group)
    return apply_fn(x, word)
