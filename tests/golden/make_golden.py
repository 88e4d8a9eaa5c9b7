"""Writes tests/golden/tiny_linear_digests.txt: SHA-256 digests of the CPU
oracle's outputs on the seeded tiny linear-layer workload (X[64,2048],
W[2048,2048]).  Calls only the oracle and the seeded input generators; the
digests catch any later, unintended change to the oracle's arithmetic.

    python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from fp8_dynamic_quantization_b200 import inputs  # noqa: E402


def digests():
    x = inputs.bf16_bits(inputs.activations_tiny())
    w = inputs.bf16_bits(inputs.weight_tiny())
    q_pt, s_pt = oracle.quant_per_tensor(x)
    q_g, s_g = oracle.quant_group128(x)
    q_w, s_w = oracle.quant_block128(w)
    R, _ = oracle.block_gemm(q_g, s_g, q_w, s_w)
    y = oracle.f64_to_bf16(R)
    out = {
        "per_tensor_scale_bits": "%08x" % np.float32(s_pt).view(np.uint32),
        "per_tensor_codes": q_pt,
        "group128_codes": q_g,
        "group128_scales": s_g,
        "block128_codes": q_w,
        "block128_scales": s_w,
        "gemm_y_bf16": y,
    }
    res = {}
    for k, v in out.items():
        res[k] = v if isinstance(v, str) else hashlib.sha256(
            np.ascontiguousarray(v).tobytes()).hexdigest()
    return res


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_linear_digests.txt")
    with open(path, "w") as f:
        f.write("# written by tests/golden/make_golden.py from the CPU oracle\n")
        for k, v in digests().items():
            f.write(f"{k} = {v}\n")
    print(open(path).read())
