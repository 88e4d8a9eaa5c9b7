"""Golden fixtures: the facts the pages state (tests/golden/page_facts.txt,
each line cited) and SHA-256 digests of the oracle's outputs on the tiny
linear-layer workload (tests/golden/tiny_linear_digests.txt, written by
tests/golden/make_golden.py, which calls only the oracle)."""
import os

import numpy as np

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_kv(name):
    out = {}
    for line in open(os.path.join(HERE, name)):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        key, val = line.split("=", 1)
        out[key.strip()] = val.split("|", 1)[0].strip()
    return out


def test_page_facts_hold_in_oracle(oracle_mod):
    f = _read_kv("page_facts.txt")
    s, e, m = int(f["e4m3_sign_bits"]), int(f["e4m3_exponent_bits"]), int(f["e4m3_mantissa_bits"])
    assert s + e + m == 8
    codes = np.arange(256, dtype=np.uint8)
    v = oracle_mod.e4m3_decode(codes)
    # the top bit is the sign; the next e bits are the exponent field: values
    # with the same exponent field share a binade (their ratio is < 2)
    for ef in range(1, 2 ** e - 1):
        block = v[ef << m:(ef + 1) << m]
        assert block.max() / block.min() < 2.0
    # the divisor of the scale is the largest finite E4M3 magnitude
    div = float(f["scale_divisor"])
    assert np.nanmax(v) == div
    assert oracle_mod.scale_from_amax(div) == 1.0
    # groups of 128 along K: one scale per group
    gk = int(f["group_size_k"])
    q, sc = oracle_mod.quant_group128(np.zeros((2, 3 * gk), np.uint16))
    assert sc.shape == (2, 3)
    assert int(f["gemm_block_k"]) == gk
    assert int(f["e4m3_widens_to_bf16_exactly"]) == 1


def test_tiny_linear_digests(oracle_mod):
    import sys
    sys.path.insert(0, HERE)
    import make_golden
    want = _read_kv("tiny_linear_digests.txt")
    got = make_golden.digests()
    assert got == want
