"""Failure detection without a GPU fault.

A device-side wait that runs out must end the kernel with FP8Q_ERR_TIMEOUT in
the library's status word (read by fp8q_device_status), write no outputs and
leave the context usable.  The wait is made to run out by a barrier that
nothing releases: the small-tensor per-tensor path's arrival count is
pre-set in the caller's workspace, so no CTA ever sees itself as the last to
arrive.  The wait is bounded by about one second of SM clock.
"""
import numpy as np
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import _abi, inputs

pytestmark = pytest.mark.gpu

FP8Q_OK, FP8Q_ERR_TIMEOUT = 0, 6


def _call(lib, x, q, s, ws):
    M, K = x.shape
    return lib.fp8_act_quant_per_tensor(x.data_ptr(), M, K, K, q.data_ptr(), K, s.data_ptr(),
                                        ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)


def test_unreleased_grid_barrier_reports_timeout(oracle_mod, cuda_lib, gpu):
    lib = _abi.load()
    M, K = 64, 2048                       # 8 CTAs: the single-launch path with a grid barrier
    x_cpu = inputs.activations_per_tensor(M, seed=31)
    x = x_cpu.to(gpu)
    q = torch.full((M, K), 0x5A, dtype=torch.uint8, device=gpu)
    s = torch.full((1,), -1.0, dtype=torch.float32, device=gpu)
    ws = torch.zeros(lib.fp8_act_quant_per_tensor_workspace_size(M, K), dtype=torch.uint8, device=gpu)
    ws.view(torch.int32)[0] = 1000        # arrival count that never reaches "last"
    fq.device_status(reset=True)

    assert _call(lib, x, q, s, ws) == FP8Q_OK          # the launch itself succeeds
    assert fq.device_status(reset=True) == FP8Q_ERR_TIMEOUT
    assert torch.all(q == 0x5A) and s.item() == -1.0   # nothing written

    # the context is still usable: a zeroed workspace gives the right answer
    ws.zero_()
    assert _call(lib, x, q, s, ws) == FP8Q_OK
    assert fq.device_status(reset=True) == FP8Q_OK
    q_ref, s_ref = oracle_mod.quant_per_tensor(inputs.bf16_bits(x_cpu))
    assert np.float32(s.item()) == s_ref
    assert np.array_equal(q.cpu().numpy(), q_ref)
