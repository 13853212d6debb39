"""The allocation-free attention backward (nc_op_attention_bwd_noalloc).

It exists for callers that cannot allocate device memory themselves; its
scratch is a fixed array inside the library.  Checked here through the C ABI
against the ordinary entry point (which takes a caller-provided scratch
buffer) on two calls in a row with different shapes, so the second call
runs on whatever the first left in the shared array; plus the size limit.
This file is collected last so a failure here comes after every other test.
"""
import numpy as np
import pytest

from pretraining_step_b200 import binding as nc
from pretraining_step_b200 import inputs

from gpu_util import dev_bf16, dev_f32, host, rel_fro, torch

pytestmark = pytest.mark.gpu


def _case(B, T, H, seed):
    t = torch()
    d = H * 128
    qkv = dev_bf16(inputs.bf16_normal(seed, (B * T, 3 * d)))
    o = dev_bf16(inputs.bf16_normal(seed + 1, (B * T, d)))
    dout = dev_bf16(inputs.bf16_normal(seed + 2, (B * T, d)))
    lse = dev_f32(np.abs(inputs.bf16_normal(seed + 3, (B, H, T))) + 2.0)
    return t, d, qkv, o, dout, lse


def _run(fn, B, T, H, case):
    t, d, qkv, o, dout, lse = case
    dq = t.empty(B * T, d, dtype=t.float32, device="cuda")
    dkv = t.zeros(B * T, 2 * d, dtype=t.bfloat16, device="cuda")
    fn(qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, o, dout, d, lse, dq, dkv[:, :d], dkv[:, d:],
       2 * d, B, T, H)
    t.cuda.synchronize()
    return host(dq), host(dkv)


def _with_caller_scratch(B, T, H):
    t = torch()
    delta = t.empty(B, H, T, dtype=t.float32, device="cuda")

    def fn(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, B_, T_, H_):
        nc.attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B_, T_, H_)
    return fn


@pytest.mark.parametrize("shapes", [((2, 200, 2), (1, 333, 3))])
def test_noalloc_matches_the_allocating_entry_point_twice(shapes):
    for i, (B, T, H) in enumerate(shapes):
        case = _case(B, T, H, 900 + 10 * i)
        dq0, dkv0 = _run(_with_caller_scratch(B, T, H), B, T, H, case)
        dq1, dkv1 = _run(nc.attention_bwd_noalloc, B, T, H, case)
        assert rel_fro(dq1, dq0) < 1e-2
        assert rel_fro(dkv1, dkv0) < 1e-2
        assert np.isfinite(dq1).all() and np.abs(dq1).max() > 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    t = torch()
    x = t.zeros(8, dtype=t.float32, device="cuda")
    with pytest.raises(nc.NcError) as e:
        # B * H * T = 2^20 + 2048 > 2^20: rejected before anything is launched.
        nc.attention_bwd_noalloc(x, x, x, 384, x, x, 128, x, x, x, x, 384, 1, 2048, 513)
    assert e.value.status == nc.NC_ERR_INVALID_ARG
    assert "scratch" in str(e.value)
