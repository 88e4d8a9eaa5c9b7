"""Guard bands around every output: the kernels write their outputs and
nothing else.

Each output is placed inside a larger device buffer filled with a canary
byte, with a band before the first byte, a band after the last, and (where
the output has a row pitch) padding at the end of every row.  After the call
every canary byte must be intact and the output must equal the same call
made into a plain buffer.  Two canary values are used, so a stray write of
one of them is still caught by the other run.  Shapes are ragged (rows and
columns off the tile sizes, short last chunks) and cover the chunked and
strided quantisation kernels (fp32 and ue8m0 group scales), the CTA-pair GEMM with its bulk-store
epilogue and split last wave, the single-CTA tiles and the swapped split-K
path.  Calls go through the C ABI with these buffers (ctypes)."""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

BAND = 4096            # bytes of canary before and after every output
CANARIES = (0xA5, 0x5A)


class Guarded:
    """A [rows, ld] output of `itemsize`-byte elements (the first `cols`
    of each row are the output) inside a canary-filled byte buffer."""

    def __init__(self, dev, rows, cols, ld, itemsize, canary):
        self.rows, self.cols, self.ld, self.itemsize = rows, cols, ld, itemsize
        nbytes = rows * ld * itemsize
        self.buf = torch.full((2 * BAND + nbytes,), canary, dtype=torch.uint8, device=dev)
        self.canary = canary

    def ptr(self):
        return self.buf.data_ptr() + BAND

    def region(self):
        return self.buf[BAND:BAND + self.rows * self.ld * self.itemsize].view(self.rows, self.ld * self.itemsize)

    def output(self):
        return self.region()[:, :self.cols * self.itemsize]

    def check(self, what):
        b = self.buf.cpu().numpy()
        assert np.all(b[:BAND] == self.canary), f"{what}: written before the output"
        assert np.all(b[-BAND:] == self.canary), f"{what}: written after the output"
        pad = self.region()[:, self.cols * self.itemsize:].cpu().numpy()
        assert np.all(pad == self.canary), f"{what}: written into the row padding"


def _lib():
    return fq.library()


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("m,k,ldq", [(4096, 7168, 7168), (1000, 1280, 1280), (300, 2048, 2048 + 64),
                                     (5, 7168, 7168 + 8)])
def test_per_tensor_quant_writes_only_its_outputs(gpu, m, k, ldq):
    lib = _lib()
    x = inputs.activations_per_tensor(m, k=k, seed=m + k).to(gpu)
    q_ref, s_ref = fq.act_quant_per_tensor(x)
    wsb = lib.fp8_act_quant_per_tensor_workspace_size(m, k)
    ws = torch.empty(wsb, dtype=torch.uint8, device=gpu)
    for canary in CANARIES:
        q = Guarded(gpu, m, k, ldq, 1, canary)
        s = Guarded(gpu, 1, 1, 1, 4, canary)
        assert lib.fp8_act_quant_per_tensor(x.data_ptr(), m, k, k, q.ptr(), ldq, s.ptr(), ws.data_ptr(), wsb,
                                            _stream()) == 0
        torch.cuda.synchronize()
        q.check("per-tensor codes")
        s.check("per-tensor scale")
        assert torch.equal(q.output(), q_ref.view(torch.uint8))
        assert torch.equal(s.output().view(torch.float32).reshape(1), s_ref)
    assert fq.device_status() == 0


@pytest.mark.parametrize("m,k,ldq", [(4096, 7168, 7168), (1000, 1280, 1280), (129, 7168, 7168),
                                     (97, 2048, 2048 + 128)])
@pytest.mark.parametrize("e8", [False, True])
def test_group128_quant_writes_only_its_outputs(gpu, m, k, ldq, e8):
    lib = _lib()
    x = inputs.activations_group(m, k=k, seed=m + k).to(gpu)
    q_ref, s_ref = fq.act_quant_group128_ue8m0(x) if e8 else fq.act_quant_group128(x)
    g = k // 128
    fn = lib.fp8_act_quant_group128_ue8m0 if e8 else lib.fp8_act_quant_group128
    for canary in CANARIES:
        q = Guarded(gpu, m, k, ldq, 1, canary)
        s = Guarded(gpu, m, g, g, 1 if e8 else 4, canary)
        assert fn(x.data_ptr(), m, k, k, q.ptr(), ldq, s.ptr(), _stream()) == 0
        torch.cuda.synchronize()
        q.check("group codes")
        s.check("group scales")
        assert torch.equal(q.output(), q_ref.view(torch.uint8))
        got = s.output().contiguous()
        if e8:
            assert torch.equal(got.reshape(m, g), s_ref.view(torch.uint8).reshape(m, g))
        else:
            assert torch.equal(got.view(torch.float32).reshape(m, g), s_ref)
    assert fq.device_status() == 0


# (M, N, K): CTA-pair tiles with a ragged edge and a split last wave (1100 x
# 3900: 80 pair tiles = 74 + 6), CTA pairs with whole waves, single-CTA
# tiles (M <= 512), swapped tiles with split-K (M <= 32)
@pytest.mark.parametrize("m,n,k", [(1100, 3900, 1024), (1280, 2048, 512), (300, 520, 512), (16, 2048, 1024)])
def test_block_gemm_writes_only_its_output(gpu, m, n, k):
    lib = _lib()
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=m + n + k)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(gpu)
    tqa, tsa, tqb, tsb = d(qa), d(sa), d(qb), d(sb)
    y_ref = fq.block_gemm(tqa.view(torch.float8_e4m3fn), tsa, tqb.view(torch.float8_e4m3fn), tsb)
    wsb = lib.fp8_block_gemm_workspace_size(m, n, k)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=gpu)
    ldy = (n + 7) // 8 * 8 + 8          # 16-byte pitch with at least 8 padding columns
    for canary in CANARIES:
        y = Guarded(gpu, m, n, ldy, 2, canary)
        assert lib.fp8_block_gemm(tqa.data_ptr(), k, tsa.data_ptr(), tqb.data_ptr(), k, tsb.data_ptr(),
                                  y.ptr(), ldy, m, n, k, ws.data_ptr(), wsb, _stream()) == 0
        torch.cuda.synchronize()
        y.check(f"GEMM {m}x{n}x{k}")
        assert torch.equal(y.output().contiguous().view(torch.int16).reshape(m, n), y_ref.view(torch.int16))
    assert fq.device_status() == 0
