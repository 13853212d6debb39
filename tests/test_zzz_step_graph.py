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
    twin model: losses and weights agree up to the order of the weight
    gradient's atomic sums."""
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
    tok_d = t.zeros((B, T), dtype=t.int32, device=dev)
    tgt_d = t.zeros((B, T), dtype=t.int32, device=dev)
    loss_a = t.zeros(1, dtype=t.float32, device=dev)
    loss_b = t.zeros(1, dtype=t.float32, device=dev)
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
            b.replay_step()
        a.sync()
        b.sync()
        la, lb = float(loss_a.item()), float(loss_b.item())
        assert abs(la - lb) <= 1e-4 * abs(la), (i, la, lb)
    assert b.launch_count() - launches0 == a.launch_count() - la0 > 0  # same kernels per step
    for i, (x, y, w0) in enumerate(zip(a.params(), b.params(), W0)):
        moved = np.linalg.norm(x.astype(np.float64) - w0)
        if moved == 0:  # wte and lm_head: not Muon's
            assert np.array_equal(x, y), i
        else:
            assert np.linalg.norm(x.astype(np.float64) - y) <= 1e-3 * moved, i
    a.close()
    b.close()
