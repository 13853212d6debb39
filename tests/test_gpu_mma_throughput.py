"""tcgen05.mma throughput by N and operand majorness (the fact the attention
kernels are designed around): an M128 x K16 MMA with both operands in shared
memory runs at the full dense rate for N >= 128 in every majorness, and at
two thirds of it for N = 64 (shared-memory operand bandwidth).  The probe
is compiled from tests/gpu_probes/mma_throughput.cu; run with -s to see the
table."""
import os
import subprocess

import pytest

from pretraining_step_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
PEAK = 8192.0  # dense bf16 FLOP per clock per SM


def test_mma_rate_by_n_and_majorness(tmp_path):
    exe = str(tmp_path / "mma_throughput")
    src = os.path.join(HERE, "gpu_probes", "mma_throughput.cu")
    subprocess.run([build.NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", build.CSRC, "-o", exe, src], check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=120).stdout
    rate = {}
    for line in out.split("\n"):
        if line.strip():
            n, a_mn, b_mn, r = line.split()
            rate[(int(n), int(a_mn), int(b_mn))] = float(r)
    for (n, a_mn, b_mn), r in sorted(rate.items()):
        print("N=%3d A %s B %s: %7.0f FLOP/clk/SM (%.1f%%)" % (
            n, "MN" if a_mn else "K ", "MN" if b_mn else "K ", r, 100 * r / PEAK))
    assert len(rate) == 9 and all(r > 0 for r in rate.values())  # no wait expired
    for key, r in rate.items():
        if key[0] >= 128:
            assert r > 0.9 * PEAK, key
    for a_mn, b_mn in ((0, 0), (0, 1), (1, 1)):
        assert rate[(64, a_mn, b_mn)] < 0.8 * rate[(128, a_mn, b_mn)]
