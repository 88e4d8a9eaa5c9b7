"""fp8_block_gemm_noalloc: the block GEMM for callers that cannot allocate
device memory (plugin hosts that hand over only input and output buffers,
serving processes that reserve the whole device pool at start-up, loops that
cannot pay for cudaMalloc/cudaFree).
Its split-K scratch is a fixed array inside the library instead of a caller
workspace.

Called through the C ABI (ctypes) on two calls in a row with different
inputs -- the second call must not see the first call's leftovers in the
shared scratch -- and checked against the oracle's float64 result within the
GEMM tolerance the other tests use, and against the allocating entry point
fp8_block_gemm.  This file is collected last
so a stop-at-first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_dynamic_quantization_b200 import _abi, inputs
import fp8_dynamic_quantization_b200 as fq

pytestmark = pytest.mark.gpu

FP8Q_OK, FP8Q_ERR_WORKSPACE = 0, 4


def _noalloc(lib, qa, sa, qb, sb, y):
    M, K = qa.shape
    N = qb.shape[0]
    return lib.fp8_block_gemm_noalloc(qa.data_ptr(), qa.stride(0), sa.data_ptr(), qb.data_ptr(),
                                      qb.stride(0), sb.data_ptr(), y.data_ptr(), y.stride(0), M, N, K,
                                      torch.cuda.current_stream().cuda_stream)


def _dev(a, gpu):
    return torch.from_numpy(np.ascontiguousarray(a)).to(gpu)


@pytest.mark.parametrize("m,n,k", [(16, 2048, 7168), (64, 7168, 7168), (3, 200, 1024)])
def test_noalloc_matches_allocating_gemm_twice(oracle_mod, cuda_lib, gpu, m, n, k):
    lib = _abi.load()
    need = lib.fp8_block_gemm_workspace_size(m, n, k)
    # these shapes split K (64 x 7168 x 7168 into more ranges than the
    # scratch holds: the call uses fewer)
    assert need > 0
    for call, seed in enumerate((101, 202)):
        qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=seed + m + n)
        tqa, tsa, tqb, tsb = (_dev(a, gpu) for a in (qa, sa, qb, sb))
        ldy = (n + 7) // 8 * 8
        y = torch.full((m, ldy), float("nan"), dtype=torch.bfloat16, device=gpu)[:, :n]
        assert _noalloc(lib, tqa, tsa, tqb, tsb, y) == FP8Q_OK
        y_ref = fq.block_gemm(tqa, tsa, tqb, tsb)
        torch.cuda.synchronize()
        Y = y.float().cpu().numpy().astype(np.float64)
        Yr = y_ref.float().cpu().numpy().astype(np.float64)
        R, T = oracle_mod.block_gemm(qa, sa, qb, sb)
        # the oracle's float64 result decides; the allocating call is a
        # second opinion (the two calls may split K differently)
        assert np.all(np.abs(Y - R) <= oracle_mod.gemm_tolerance(R, T)), f"call {call}: outside the oracle's tolerance"
        assert np.all(np.abs(Y - Yr) <= oracle_mod.gemm_tolerance(Yr, T)), f"call {call}: differs from fp8_block_gemm"
    assert fq.device_status() == 0


def test_noalloc_cuts_the_split_tail_to_its_scratch(oracle_mod, cuda_lib, gpu):
    """4000 x 7100 x 4608 leaves a short last wave whose tiles the GEMM splits
    along K; the allocating call's split needs more than the fixed scratch,
    so this call splits them fewer ways.  Tiles outside that wave are
    computed the same way by both calls (same bytes); the split tiles are
    checked against the oracle's tolerance.  Two calls in a row."""
    lib = _abi.load()
    m, n, k = 4000, 7100, 4608
    assert lib.fp8_block_gemm_workspace_size(m, n, k) > _abi.NOALLOC_MAX_SCRATCH_BYTES
    sms = torch.cuda.get_device_properties(gpu).multi_processor_count
    plan = (ctypes.c_int * 11)()
    ws = ctypes.c_size_t(0)
    assert lib.fp8q_gemm_plan(m, n, k, sms, ctypes.c_size_t(-1).value, plan, ctypes.byref(ws)) == FP8Q_OK
    pair, bn, tiles_p, tiles_q, tail = plan[1], plan[2], plan[5], plan[6], plan[9]
    rows = 256 if pair else 128               # a CTA pair computes 256-row tiles
    assert tiles_p == -(-m // rows) and tiles_q == -(-n // bn)
    assert tail == (tiles_p * tiles_q) % (sms // 2 if pair else sms) and tail > 0
    in_tail = np.zeros((m, n), dtype=bool)
    for t in range(tiles_p * tiles_q - tail, tiles_p * tiles_q):
        tp, tq = t % tiles_p, t // tiles_p
        in_tail[tp * rows:tp * rows + rows, tq * bn:tq * bn + bn] = True
    ms, ns = np.nonzero(in_tail)
    for seed in (303, 404):
        qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=seed)
        tqa, tsa, tqb, tsb = (_dev(a, gpu) for a in (qa, sa, qb, sb))
        ldy = (n + 7) // 8 * 8                 # 16-byte row pitch
        y = torch.full((m, ldy), float("nan"), dtype=torch.bfloat16, device=gpu)[:, :n]
        assert _noalloc(lib, tqa, tsa, tqb, tsb, y) == FP8Q_OK
        y_ref = fq.block_gemm(tqa, tsa, tqb, tsb)
        torch.cuda.synchronize()
        Y = y.float().cpu().numpy().astype(np.float64)
        Yr = y_ref.float().cpu().numpy().astype(np.float64)
        assert np.array_equal(Y[~in_tail], Yr[~in_tail])
        R, T = oracle_mod.block_gemm_points(qa, sa, qb, sb, ms, ns)
        assert np.all(np.abs(Y[ms, ns] - R) <= oracle_mod.gemm_tolerance(R, T)), f"seed {seed}"
    assert fq.device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_lib, gpu):
    """32 tokens run with the operands swapped, and with K = 8320 (65 K
    blocks) that launch needs at least two K ranges: 2 * 32 * 32776 * 4
    bytes, just over the scratch.  Refused before anything is enqueued (the
    buffers are full-size all the same)."""
    lib = _abi.load()
    m, n, k = 32, 32776, 8320
    assert lib.fp8_block_gemm_workspace_size(m, n, k) > _abi.NOALLOC_MAX_SCRATCH_BYTES
    qa = torch.zeros(m, k, dtype=torch.uint8, device=gpu)
    sa = torch.ones(m, k // 128, dtype=torch.float32, device=gpu)
    qb = torch.zeros(n, k, dtype=torch.uint8, device=gpu)
    sb = torch.ones((n + 127) // 128, k // 128, dtype=torch.float32, device=gpu)
    y = torch.full((m, n), 3.0, dtype=torch.bfloat16, device=gpu)
    assert _noalloc(lib, qa, sa, qb, sb, y) == FP8Q_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)                 # nothing was enqueued
