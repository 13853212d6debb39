"""The training step captured as one CUDA graph (nc_step_capture /
nc_step_replay) against the same calls made eagerly."""
import numpy as np
import pytest

from pretraining_step_b200 import binding as nc
from pretraining_step_b200 import inputs

from gpu_util import torch

pytestmark = pytest.mark.gpu


def _gpt(depth, **kw):
    return nc.GPT(depth, vocab=32768, **kw)


def test_step_graph_matches_eager_steps():
    """A captured step (fwd + bwd + Muon as one CUDA graph) replayed over
    three batches written in place matches the same calls made eagerly on a
    twin model.  The step is not bitwise deterministic: the weight-gradient
    split-K sums, the attention dQ sums, the embedding scatter and Muon's
    squared norms are fp32 atomics whose order varies, and Newton-Schulz
    magnifies that noise along small singular directions.  So a third model,
    an eager twin of the first, measures the spread two eager runs show, and
    the graph must stay within a small multiple of it."""
    t = torch()
    depth, B, T, lr, mu = 2, 2, 128, 0.02, 0.95
    s = t.cuda.Stream()
    dev = t.device("cuda")
    # One eager step of a throwaway model first, so every kernel of the step
    # has been loaded and configured before anything is captured.
    w = _gpt(depth, seed=30, all_random=True, stream=s)
    tk, tg = inputs.token_batch(30, B, T)
    w.fwd_bwd(tk, tg)
    w.muon_step(lr, mu)
    w.sync()
    w.close()
    a = _gpt(depth, seed=31, all_random=True, stream=s)
    b = _gpt(depth, seed=31, all_random=True, stream=s)
    c = _gpt(depth, seed=31, all_random=True, stream=s)  # eager control
    tok_d = t.zeros((B, T), dtype=t.int32, device=dev)
    tgt_d = t.zeros((B, T), dtype=t.int32, device=dev)
    loss_a = t.zeros(1, dtype=t.float32, device=dev)
    loss_b = t.zeros(1, dtype=t.float32, device=dev)
    loss_c = t.zeros(1, dtype=t.float32, device=dev)
    t.cuda.synchronize()
    launches0 = b.launch_count()
    b.capture_step(tok_d, tgt_d, loss_b, lr, mu)
    assert b.launch_count() == launches0  # recorded, not run
    W0 = a.params()
    assert all(np.array_equal(x, y) for x, y in zip(W0, b.params()))  # nothing ran
    la0 = a.launch_count()
    for i in range(3):
        tk, tg = inputs.token_batch(32 + i, B, T)
        with t.cuda.stream(s):
            tok_d.copy_(t.from_numpy(tk))
            tgt_d.copy_(t.from_numpy(tg))
            a.fwd_bwd_async(tok_d, tgt_d, loss_a)
            a.muon_step(lr, mu)
            c.fwd_bwd_async(tok_d, tgt_d, loss_c)
            c.muon_step(lr, mu)
            b.replay_step()
        a.sync()
        b.sync()
        c.sync()
        la, lb, lc = float(loss_a.item()), float(loss_b.item()), float(loss_c.item())
        assert abs(la - lb) <= max(3 * abs(la - lc), 1e-4 * abs(la)), (i, la, lb, lc)
    assert b.launch_count() - launches0 == a.launch_count() - la0 > 0  # same kernels per step
    diff, spread = 0.0, 0.0
    for i, (x, y, z, w0) in enumerate(zip(a.params(), b.params(), c.params(), W0)):
        x = x.astype(np.float64)
        moved = np.linalg.norm(x - w0)
        if moved == 0:  # wte and lm_head: not Muon's
            assert np.array_equal(x, y) and np.array_equal(x, z), i
            continue
        diff = max(diff, np.linalg.norm(x - y) / moved)
        spread = max(spread, np.linalg.norm(x - z) / moved)
    assert spread < 0.1, spread  # the eager noise itself stays small
    assert diff <= max(3 * spread, 1e-3), (diff, spread)
    a.close()
    b.close()
    c.close()
