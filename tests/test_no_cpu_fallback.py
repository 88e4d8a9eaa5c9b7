"""Every public operation of the Python binding refuses host tensors with an
error: nothing is computed on the CPU, so a missing GPU or a tensor on the
wrong device can never fall back to a host implementation."""
import pytest
import torch

import fp8_dynamic_quantization_b200 as fq

M, N, K = 4, 256, 256
G = K // 128


def _x():
    return torch.randn(M, K).to(torch.bfloat16)


def _w():
    return torch.randn(N, K).to(torch.bfloat16)


def _codes(rows):
    return torch.zeros(rows, K, dtype=torch.uint8)


CASES = {
    "act_quant_per_tensor": lambda: fq.act_quant_per_tensor(_x()),
    "act_amax": lambda: fq.act_amax(_x()),
    "act_quant_apply": lambda: fq.act_quant_apply(_x(), torch.zeros(1, dtype=torch.int32)),
    "act_quant_group128": lambda: fq.act_quant_group128(_x()),
    "weight_quant_block128": lambda: fq.weight_quant_block128(_w()),
    "act_quant_per_channel": lambda: fq.act_quant_per_channel(_x()),
    "act_quant_group128_ue8m0": lambda: fq.act_quant_group128_ue8m0(_x()),
    "weight_quant_block128_ue8m0": lambda: fq.weight_quant_block128_ue8m0(_w()),
    "block_gemm": lambda: fq.block_gemm(_codes(M), torch.ones(M, G), _codes(N), torch.ones(N // 128, G)),
    "gemm_per_tensor": lambda: fq.gemm_per_tensor(_codes(M), torch.ones(1), _codes(N), torch.ones(1)),
    "gemm_per_channel": lambda: fq.gemm_per_channel(_codes(M), torch.ones(M), _codes(N), torch.ones(N)),
    "block_gemm_ue8m0": lambda: fq.block_gemm_ue8m0(_codes(M), torch.full((M, G), 127, dtype=torch.uint8),
                                                    _codes(N), torch.full((N // 128, G), 127, dtype=torch.uint8)),
    "linear": lambda: fq.linear(_x(), _codes(N), torch.ones(N // 128, G)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_host_tensors_are_refused(cuda_lib, name):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        CASES[name]()
