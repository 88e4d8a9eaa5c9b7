"""Every GEMM launch mode against the oracle, forced through the tuning
override FP8Q_GEMM_TILE (read once per process, hence one child process per
mode).  The default launch table only selects some of them."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import oracle
import fp8_dynamic_quantization_b200 as fq
from fp8_dynamic_quantization_b200 import inputs
dev = torch.device("cuda:0")
shapes = [tuple(int(v) for v in s.split("x")) for s in sys.argv[3].split(",")]
for m, n, k in shapes:
    qa, sa, qb, sb = inputs.gemm_operands(m, n, k, seed=m + n + k)
    y = fq.block_gemm(torch.from_numpy(qa).to(dev), torch.from_numpy(sa).to(dev),
                      torch.from_numpy(qb).to(dev), torch.from_numpy(sb).to(dev))
    R, T = oracle.block_gemm(qa, sa, qb, sb)
    Y = y.float().cpu().numpy().astype(np.float64)
    bad = int((np.abs(Y - R) > oracle.gemm_tolerance(R, T)).sum())
    assert bad == 0, (m, n, k, bad)
    # per-tensor scales (pair rows run the pair kernel here too)
    s_a, s_b = np.float32(0.05), np.float32(0.003)
    y = fq.gemm_per_tensor(torch.from_numpy(qa).to(dev), torch.tensor([s_a], device=dev),
                           torch.from_numpy(qb).to(dev), torch.tensor([s_b], device=dev))
    R, T = oracle.gemm_per_tensor(qa, s_a, qb, s_b)
    Y = y.float().cpu().numpy().astype(np.float64)
    bad = int((np.abs(Y - R) > oracle.gemm_tolerance(R, T)).sum())
    assert bad == 0, ("per-tensor", m, n, k, bad)
    # ue8m0 scales applied by the tensor cores
    g = np.random.default_rng(m + n)
    ea = g.integers(115, 135, sa.shape).astype(np.uint8)
    eb = g.integers(115, 135, sb.shape).astype(np.uint8)
    y = fq.block_gemm_ue8m0(torch.from_numpy(qa).to(dev), torch.from_numpy(ea).to(dev),
                            torch.from_numpy(qb).to(dev), torch.from_numpy(eb).to(dev))
    R, T = oracle.gemm_ue8m0(qa, ea, qb, eb)
    Y = y.float().cpu().numpy().astype(np.float64)
    bad = int((np.abs(Y - R) > oracle.gemm_tolerance(R, T)).sum())
    assert bad == 0, ("ue8m0", m, n, k, bad)
    # per-channel scales applied in the epilogue
    ra = g.uniform(1e-3, 1e-1, m).astype(np.float32)
    rb = g.uniform(1e-3, 1e-1, n).astype(np.float32)
    y = fq.gemm_per_channel(torch.from_numpy(qa).to(dev), torch.from_numpy(ra).to(dev),
                            torch.from_numpy(qb).to(dev), torch.from_numpy(rb).to(dev))
    R, T = oracle.gemm_per_channel(qa, ra, qb, rb)
    Y = y.float().cpu().numpy().astype(np.float64)
    bad = int((np.abs(Y - R) > oracle.gemm_tolerance(R, T)).sum())
    assert bad == 0, ("per-channel", m, n, k, bad)
assert fq.device_status() == 0
print("ok")
'''


def _run_child(tile, shapes):
    env = dict(os.environ, FP8Q_GEMM_TILE=tile)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, tile, shapes], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


@pytest.mark.parametrize("tile", ["normal:128", "normal:192", "normal:256", "pair:256", "pair:128",
                                  "swap:16", "swap:32", "swap:64", "swap:128:3"])
def test_gemm_mode_matches_oracle(gpu, cuda_lib, oracle_mod, tile):
    # 257 x 384 x 640: five K blocks, so the last two-K-block round of a CTA
    # pair's 256 x 128 tiles holds one
    _run_child(tile, "1x200x256,130x300x512,600x520x1280,1025x264x256,257x384x640")


# Shapes whose tile count leaves a short last wave on a 148-SM part, so the
# tail tiles are split along K and summed by tail_reduce_kernel:
#   1280 x 3840: pair 256 x 256 -> 75 tiles = 74 + 1; pair 256 x 128 -> 150 =
#                2 x 74 + 2; 128 x 256 -> 150 = 148 + 2
#   1100 x 3900 (ragged rows and columns): pair 256 x 256 -> 80 = 74 + 6;
#                pair 256 x 128 -> 155 = 2 x 74 + 7
#   1280 x 3840 x 1152: nine K blocks split into 4 ranges (2, 2, 2, 3 blocks)
@pytest.mark.parametrize("tile", ["pair:256", "pair:128", "normal:256"])
def test_split_last_wave_matches_oracle(gpu, cuda_lib, oracle_mod, tile):
    _run_child(tile, "1280x3840x1024,1100x3900x1024,1280x3840x1152")
