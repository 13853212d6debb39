"""The allocation-free attention backward (nc_op_attention_bwd_noalloc).

It serves callers that cannot allocate device memory themselves; its only
scratch, the row sums D = rowsum(dO * O), lives in a fixed array inside the
library.  Checked here through the C ABI on two calls in a row, the larger
shape first, so the second call runs over entries the first one left in the
shared array: each call against the oracle's backward (from the oracle's O
and lse), and against the ordinary entry point, which takes a
caller-provided scratch buffer: dK and dV bit for bit (they accumulate in a
fixed order), dQ (fp32 atomic sums in varying order) within the oracle bar.
Plus the size limit.  This file is collected last, so a failure here comes
after every other test has run.
"""
import numpy as np
import pytest

import oracle
from pretraining_step_b200 import binding as nc
from pretraining_step_b200 import inputs

from gpu_util import dev_bf16, dev_f32, host, rel_fro, torch

pytestmark = pytest.mark.gpu


def _case(B, T, H, seed):
    """q, k, v from the seeded generator; O and lse from the oracle's forward
    (O rounded to bf16 like the saved activation); a seeded dO."""
    d = H * 128
    qkv = inputs.bf16_normal(seed, (B * T, 3 * d))
    q = qkv[:, :d].reshape(B, T, H, 128)
    k = qkv[:, d:2 * d].reshape(B, T, H, 128)
    v = qkv[:, 2 * d:].reshape(B, T, H, 128)
    oref, lref, _ = oracle.attention(q, k, v)
    o_b = inputs.round_to_bf16(oref.reshape(B * T, d).astype(np.float32))
    dout = inputs.bf16_normal(seed + 1, (B * T, d))
    ref = oracle.attention_bwd(q, k, v, lref, dout.reshape(B, T, H, 128))
    dev = (dev_bf16(qkv), dev_bf16(o_b), dev_bf16(dout), dev_f32(lref.astype(np.float32)))
    return d, dev, [r.reshape(B * T, d) for r in ref]


def _run(fn, B, T, H, d, dev):
    t = torch()
    qkv, o, dout, lse = dev
    dq = t.empty(B * T, d, dtype=t.float32, device="cuda")
    dkv = t.zeros(B * T, 2 * d, dtype=t.bfloat16, device="cuda")
    fn(qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, o, dout, d, lse, dq, dkv[:, :d], dkv[:, d:],
       2 * d, B, T, H)
    nc.op_sync()
    return host(dq), host(dkv[:, :d]), host(dkv[:, d:])


def _with_caller_scratch(B, T, H):
    t = torch()
    delta = t.empty(B, H, T, dtype=t.float32, device="cuda")

    def fn(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, B_, T_, H_):
        nc.attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B_, T_, H_)
    return fn


def test_noalloc_matches_the_oracle_and_the_allocating_entry_point_twice():
    # The larger call first: the second, smaller one runs over stale entries.
    for i, (B, T, H) in enumerate([(2, 333, 3), (1, 200, 2)]):
        d, dev, (rq, rk, rv) = _case(B, T, H, 900 + 10 * i)
        dq1, dk1, dv1 = _run(nc.attention_bwd_noalloc, B, T, H, d, dev)
        assert rel_fro(dq1, rq) < 1e-2
        assert rel_fro(dk1, rk) < 1e-2
        assert rel_fro(dv1, rv) < 1e-2
        dq0, dk0, dv0 = _run(_with_caller_scratch(B, T, H), B, T, H, d, dev)
        assert np.array_equal(dk1, dk0) and np.array_equal(dv1, dv0)
        assert rel_fro(dq1, dq0) < 1e-2


def test_noalloc_rejects_sizes_beyond_its_scratch():
    t = torch()
    x = t.zeros(8, dtype=t.float32, device="cuda")
    with pytest.raises(nc.NcError) as e:
        # B * H * T = 2^20 + 2048 > 2^20: rejected before anything is launched.
        nc.attention_bwd_noalloc(x, x, x, 384, x, x, 128, x, x, x, x, 384, 1, 2048, 513)
    assert e.value.status == nc.NC_ERR_INVALID_ARG
    assert "scratch" in str(e.value)
