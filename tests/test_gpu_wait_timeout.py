"""Failure detection without a fault: a bounded device wait that runs out.

A kernel waits, through the library's tc::mbar_wait, on an mbarrier that
nothing arrives on.  After the wall-clock limit (2 s) the wait records the
timeout in the device status word and the kernel returns; the launch
completes without a CUDA error, the host reads the status, and the next
kernel runs normally.  The probe is compiled from
tests/gpu_probes/wait_timeout.cu."""
import os
import subprocess

import pytest

from pretraining_step_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
DEV_TIMEOUT = 1   # status word value of an expired wait
LIMIT_MS = 2000.0  # the wait's wall-clock limit


def test_expired_wait_reports_status_and_leaves_the_context_usable(tmp_path):
    exe = str(tmp_path / "wait_timeout")
    src = os.path.join(HERE, "gpu_probes", "wait_timeout.cu")
    subprocess.run([build.NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", build.CSRC, "-o", exe, src], check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60).stdout
    status, waited_ok, ms, after = out.split()
    assert int(status) == DEV_TIMEOUT
    assert int(waited_ok) == 0          # the wait gave up
    assert 0.95 * LIMIT_MS <= float(ms) < 3 * LIMIT_MS  # (the device timer's own granularity)
    assert int(after) == 1              # the next kernel ran
