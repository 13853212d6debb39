"""Failure detection and recovery without a GPU fault.

- A kernel waits, through the library's tc::mbar_wait, on an mbarrier that
  nothing arrives on.  After the wall-clock limit (2 s) the wait records the
  timeout in the device status word and the kernel returns; the launch
  completes without a CUDA error, the host reads the status, and the next
  kernel runs normally (probe: tests/gpu_probes/wait_timeout.cu).
- A timeout code planted in a handle's status word surfaces as
  NC_ERR_TIMEOUT and poisons the handle.
- An activation request far beyond the device's memory returns NC_ERR_OOM
  and the handle keeps working."""
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


def test_planted_timeout_status_poisons_the_handle():
    """Host side of the same path: a timeout code in the status word (planted
    here instead of produced by a stuck kernel) surfaces as NC_ERR_TIMEOUT
    at the next synchronising call, and the handle then refuses work."""
    import numpy as np
    from pretraining_step_b200 import binding as nc
    from pretraining_step_b200 import inputs

    from gpu_util import torch
    t = torch()
    m = nc.GPT(2, vocab=512, seed=3)
    ptr = nc.lib().nc_debug_status_word(m.h)
    assert ptr

    class _Word:
        __cuda_array_interface__ = {"shape": (1,), "typestr": "<i4", "data": (ptr, False),
                                    "version": 3}

    word = t.as_tensor(_Word(), device="cuda")  # aliases the status word
    m.sync()                                      # no error yet
    word.fill_(DEV_TIMEOUT)
    t.cuda.synchronize()
    with pytest.raises(nc.NcError) as e:
        m.sync()
    assert e.value.status == nc.NC_ERR_TIMEOUT
    tok, tgt = inputs.token_batch(4, 1, 16, vocab=512)
    with pytest.raises(nc.NcError) as e:
        m.fwd_bwd(tok, tgt)
    assert e.value.status == nc.NC_ERR_TIMEOUT
    assert np.isfinite(m.read(0)).all()  # the parameters are still readable
    m.close()


def test_activation_request_beyond_memory_is_oom_and_the_handle_recovers():
    """B*T = 2^24 tokens at vocabulary 32768 asks for over a terabyte of
    activations (the bf16 logits alone are 1 TiB): the allocation fails, the
    call returns NC_ERR_OOM before touching the device, and a normal step on
    the same handle then succeeds."""
    import numpy as np
    from pretraining_step_b200 import binding as nc
    from pretraining_step_b200 import inputs

    m = nc.GPT(2, seed=5)
    big = np.zeros((4096, 4096), dtype=np.int32)
    with pytest.raises(nc.NcError) as e:
        m.fwd_bwd(big, big)
    assert e.value.status == nc.NC_ERR_OOM
    tok, tgt = inputs.token_batch(6, 1, 64)
    loss = m.fwd_bwd(tok, tgt)
    assert abs(loss - np.log(32768)) < 1e-3  # specified init: zero lm_head
    m.close()
