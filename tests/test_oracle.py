"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: published
test values, closed forms, invariants, finite differences, or a brute-force
computation written independently here.  A plausible slip in the oracle (a
dropped term, a sign, a swapped index or operand) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from pretraining_step_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
V_SMALL = 64


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ RNG, shapes
def test_splitmix64_published_values():
    g = _golden("splitmix64.json")
    for s, o in zip(g["inputs_state_before_step"], g["outputs"]):
        assert oracle.splitmix64(int(s, 16)) == int(o, 16)
        assert int(inputs.splitmix64(np.uint64(int(s, 16)))) == int(o, 16)


@pytest.mark.parametrize("depth", [4, 12, 20, 26])
def test_shapes_from_depth(depth):
    g = _golden("model_pins.json")["depth%d" % depth]
    s = oracle.dims(depth)
    assert (s["d"], s["n_head"], s["mlp"], s["head_dim"]) == (g["d"], g["n_head"], g["mlp"], 128)
    block = sum(oracle.param_numel(depth, i) for i in range(1, 6 * depth + 1))
    assert block == g["block_params"]
    if "lm_head_params" in g:
        assert oracle.param_numel(depth, 6 * depth + 1) == g["lm_head_params"]
        assert oracle.param_numel(depth, 0) == g["wte_params"]


def test_depth_one_has_one_head_of_width_64():
    s = oracle.dims(1)
    assert (s["d"], s["n_head"], s["head_dim"]) == (64, 1, 64)
    with pytest.raises(ValueError):
        oracle.dims(3)  # d = 192 is not a whole number of 128-wide heads


def test_init_statistics_and_zero_pattern():
    depth = 4
    P = oracle.init_params(depth, 32768, seed=7, spec_zero=True)
    shapes = oracle.param_shapes(depth)
    assert [p.shape for p in P] == shapes
    for i, p in enumerate(P):
        if i == len(P) - 1 or (i > 0 and (i - 1) % 6 in (3, 5)):
            assert not p.any(), "out-projections and lm_head start at zero"
            continue
        fan_in = 1 if i == 0 else shapes[i][1]
        std = fan_in ** -0.5
        x = p.astype(np.float64) / std
        n = x.size
        assert abs(x.mean()) < 5 / math.sqrt(n)
        assert abs(x.std() - 1) < 6 / math.sqrt(2 * n)
    # Box-Muller normals: kurtosis 3 and symmetric tails on the big table.
    x = P[0].astype(np.float64).ravel()
    k = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    assert abs(k - 3) < 0.02
    assert abs(np.mean(x > 1.0) - 0.158655) < 2e-3
    # Deterministic and seed-dependent.
    Q = oracle.init_params(depth, 32768, seed=7, spec_zero=True)
    R = oracle.init_params(depth, 32768, seed=8, spec_zero=True)
    assert np.array_equal(P[1], Q[1]) and not np.array_equal(P[1], R[1])
    A = oracle.init_params(depth, 32768, seed=7, spec_zero=False)
    assert np.array_equal(A[1], P[1]) and A[4].any() and A[-1].any()
    assert abs(A[-1].std() * math.sqrt(256) - 1) < 0.01


# ------------------------------------------------------------------ RMSNorm, RoPE
def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 96)) * np.array([[1e-4], [0.1], [1], [10], [1e3]])
    y, r = oracle.rmsnorm(x)
    m = np.mean(x * x, axis=1)
    # mean(y^2) = m / (m + eps) exactly, and y is x scaled per row.
    np.testing.assert_allclose(np.mean(y * y, axis=1), m / (m + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(y / x, np.broadcast_to(r[:, None], x.shape), rtol=1e-12)
    z, _ = oracle.rmsnorm(np.zeros((1, 8)))
    assert not z.any()


def test_rope_two_dim_rotation_is_by_pos_radians():
    for p in [0, 1, 2, 7, 1000]:
        v = oracle.rope_row(np.array([1.0, 0.0]), p)
        np.testing.assert_allclose(v, [math.cos(p), math.sin(p)], atol=1e-15)


def test_rope_pairing_and_frequency():
    hd, p, i = 128, 37, 5
    e = np.zeros(hd)
    e[i] = 1.0
    v = oracle.rope_row(e, p)
    th = p * 10000.0 ** (-2.0 * i / hd)
    expect = np.zeros(hd)
    expect[i], expect[i + 64] = math.cos(th), math.sin(th)
    np.testing.assert_allclose(v, expect, atol=1e-14)


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    assert np.array_equal(oracle.rope_row(q, 0), q)
    for m, n in [(5, 2), (100, 3), (2047, 2000)]:
        qm = oracle.rope_row(q, m)
        assert abs(np.linalg.norm(qm) - np.linalg.norm(q)) < 1e-12
        a = qm @ oracle.rope_row(k, n)
        b = oracle.rope_row(q, m + 11) @ oracle.rope_row(k, n + 11)
        assert abs(a - b) < 1e-11


# ------------------------------------------------------------------ attention
def _brute_attention(q, k, v):
    B, T, H, hd = q.shape
    o = np.zeros_like(q)
    lse = np.zeros((B, H, T))
    for b in range(B):
        for h in range(H):
            s = q[b, :, h, :] @ k[b, :, h, :].T / math.sqrt(hd)
            s = np.where(np.tril(np.ones((T, T))) > 0, s, -np.inf)
            mx = s.max(axis=1, keepdims=True)
            e = np.exp(s - mx)
            lse[b, h] = (mx[:, 0] + np.log(e.sum(axis=1)))
            o[b, :, h, :] = (e / e.sum(axis=1, keepdims=True)) @ v[b, :, h, :]
    return o, lse


def test_attention_against_brute_force_and_row_sums():
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((2, 9, 3, 16)) for _ in range(3))
    o, lse, P = oracle.attention(q, k, v, want_probs=True)
    ob, lb = _brute_attention(q, k, v)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12)
    np.testing.assert_allclose(P.sum(axis=-1), 1.0, rtol=1e-13)
    assert not np.triu(P, k=1).any()


def test_attention_special_cases():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, 6, 2, 8))
    # T = 1: the only key is the query's own position, so o = v.
    o1, lse1, _ = oracle.attention(v[:, :1], v[:, :1] * 2, v[:, :1])
    np.testing.assert_allclose(o1, v[:, :1], rtol=1e-14)
    # q = 0: uniform weights over the causal prefix, o_t = mean(v_0..t), lse = ln(t+1).
    o, lse, _ = oracle.attention(np.zeros_like(v), rng.standard_normal(v.shape), v)
    expect = np.cumsum(v, axis=1) / np.arange(1, 7)[None, :, None, None]
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, 7)), rtol=1e-14)


# ------------------------------------------------------------------ whole model
def test_loss_at_spec_init_is_ln_vocab_and_gradients_closed_form():
    depth, B, T = 2, 2, 16
    g = _golden("model_pins.json")
    P = oracle.init_params(depth, 32768, seed=3, spec_zero=True)
    tok, tgt = inputs.token_batch(5, B, T)
    loss, G, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt)
    assert abs(loss - g["ln_vocab"]) < 1e-12
    assert abs(loss - 15 * math.log(2)) < 1e-12
    for i in range(len(G) - 1):
        assert not G[i].any(), "every gradient except lm_head's is exactly zero"
    # dW_lm = sum_n (1/V - onehot(target_n))^T rms(E[token_n]) / N
    N, V = B * T, 32768
    x = P[0][tok.ravel()].astype(np.float64)
    xf = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6)
    expect = np.tile(xf.sum(axis=0) / (V * N), (V, 1))
    np.subtract.at(expect, tgt.ravel(), xf / N)
    np.testing.assert_allclose(G[-1], expect, rtol=1e-10, atol=1e-15)


def test_loss_near_ln_vocab_with_small_head():
    depth = 2
    P = inputs.random_params(depth, seed=4, head_std=1e-4)
    tok, tgt = inputs.token_batch(6, 1, 32)
    loss, _, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, grads=False)
    assert abs(loss - math.log(32768)) < 5e-3


def test_causality_exact():
    depth, T, t0 = 2, 10, 6
    P = inputs.random_params(depth, seed=5, vocab=V_SMALL)
    tok, tgt = inputs.token_batch(7, 1, T, vocab=V_SMALL)
    _, _, z0 = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, grads=False, want_logits=True)
    tok2 = tok.copy()
    tok2[0, t0] = (tok2[0, t0] + 1) % V_SMALL
    _, _, z1 = oracle.gpt_fwd_bwd(depth, P, tok2, tgt, vocab=V_SMALL, grads=False,
                                  want_logits=True)
    assert np.array_equal(z0[:t0], z1[:t0]), "positions before t0 must not see token t0"
    assert not np.allclose(z0[t0:], z1[t0:])


def test_accumulation_invariant():
    """One batch of B rows gives the mean of the gradients of its rows (the
    single-GPU gradient-accumulation equivalence the pages describe)."""
    depth, B, T = 1, 4, 8
    P = inputs.random_params(depth, seed=8, vocab=V_SMALL)
    tok, tgt = inputs.token_batch(9, B, T, vocab=V_SMALL)
    loss, G, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL)
    acc = [np.zeros_like(g) for g in G]
    tot = 0.0
    for b in range(B):
        lb, Gb, _ = oracle.gpt_fwd_bwd(depth, P, tok[b:b + 1], tgt[b:b + 1], vocab=V_SMALL)
        tot += lb / B
        for a, g in zip(acc, Gb):
            a += g / B
    assert abs(loss - tot) < 1e-12
    for a, g in zip(acc, G):
        np.testing.assert_allclose(g, a, rtol=1e-9, atol=1e-13)


@pytest.mark.parametrize("depth", [1, 2])
def test_gradients_central_finite_differences(depth):
    """Central differences on a depth-1 (one 64-wide head) and a depth-2 (one
    128-wide head) model at T = 8 and a 64-entry vocabulary, every tensor."""
    T = 8
    P = inputs.random_params(depth, seed=10 + depth, vocab=V_SMALL, head_std=0.5)
    tok, tgt = inputs.token_batch(11, 1, T, vocab=V_SMALL)
    _, G, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL)
    rng = np.random.default_rng(12)
    h = 2.0 ** -12
    for ti, (p, g) in enumerate(zip(P, G)):
        scale = np.abs(g).max()
        assert scale > 0, "tensor %d has an all-zero gradient" % ti
        # Pick the largest-gradient coordinate plus random ones.
        picks = [np.unravel_index(np.argmax(np.abs(g)), g.shape)]
        picks += [tuple(rng.integers(0, s) for s in g.shape) for _ in range(3)]
        if ti == 0:
            picks = [(int(tok[0, j]), int(rng.integers(0, p.shape[1]))) for j in range(3)]
            picks.append(np.unravel_index(np.argmax(np.abs(g)), g.shape))
        for idx in picks:
            w0 = p[idx]
            Pp = [q.copy() for q in P]
            Pm = [q.copy() for q in P]
            Pp[ti][idx] = np.float32(w0 + h)
            Pm[ti][idx] = np.float32(w0 - h)
            lp, _, _ = oracle.gpt_fwd_bwd(depth, Pp, tok, tgt, vocab=V_SMALL, grads=False)
            lm, _, _ = oracle.gpt_fwd_bwd(depth, Pm, tok, tgt, vocab=V_SMALL, grads=False)
            fd = (lp - lm) / (float(Pp[ti][idx]) - float(Pm[ti][idx]))
            assert abs(fd - g[idx]) <= 2e-5 * scale + 1e-9, (ti, idx, fd, g[idx], scale)


# ------------------------------------------------------------------ Newton-Schulz, Muon
def _f(x, a=3.4445, b=-4.7750, c=2.0315):
    return a * x + b * x ** 3 + c * x ** 5


def _orth(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


@pytest.mark.parametrize("shape", [(24, 24), (16, 40), (40, 16)])
def test_newton_schulz_acts_on_singular_values_by_the_quintic(shape):
    m, n = shape
    k = min(m, n)
    rng = np.random.default_rng(13)
    U, Vt = _orth(rng, m)[:, :k], _orth(rng, n)[:k, :]
    sig = np.geomspace(1.0, 0.01, k)
    G = (U * sig) @ Vt
    out = oracle.newton_schulz(G)
    s = sig / (np.linalg.norm(sig) + 1e-7)
    for _ in range(5):
        s = _f(s)
    np.testing.assert_allclose(out, (U * s) @ Vt, rtol=0, atol=1e-12)


def test_newton_schulz_left_and_right_forms_agree():
    rng = np.random.default_rng(14)
    for m, n in [(12, 30), (30, 12)]:
        G = rng.standard_normal((m, n))
        X = G / (np.linalg.norm(G) + 1e-7)
        for _ in range(5):
            A = X @ X.T
            B = -4.7750 * A + 2.0315 * (A @ A)
            X = 3.4445 * X + B @ X
        np.testing.assert_allclose(oracle.newton_schulz(G), X, rtol=0, atol=1e-12)


def test_newton_schulz_singular_values_in_band():
    G = inputs.normal_stack(15, 1, 64, 256, bf16_exact=False)[0]
    s = np.linalg.svd(oracle.newton_schulz(G), compute_uv=False)
    assert s.min() > 0.6 and s.max() < 1.21


def test_muon_update_momentum_and_apply():
    rng = np.random.default_rng(16)
    W, M, G = (rng.standard_normal((20, 48)) for _ in range(3))
    lr, mu = 0.02, 0.95
    W1, M1 = oracle.muon_update(W, M, G, lr, mu)
    np.testing.assert_array_equal(M1, mu * M + G)
    np.testing.assert_allclose((W - W1) / lr, oracle.newton_schulz(mu * M + G), atol=1e-10)


# ------------------------------------------------------------------ windowed / grouped-KV attention
def _qkv(seed, B, T, H, Hkv, hd):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, H, hd)), rng.standard_normal((B, T, Hkv, hd)),
            rng.standard_normal((B, T, Hkv, hd)))


@pytest.mark.parametrize("window", [-1, 9, 40])
def test_attention_ex_without_groups_or_window_is_the_causal_oracle(window):
    """Hkv = H and a window reaching back past the row start reduce it to the
    pinned full-causal oracle, forward and backward."""
    B, T, H, hd = 2, 9, 3, 8
    q, k, v = _qkv(60, B, T, H, H, hd)
    o, lse = oracle.attention_ex(q, k, v, window=window)
    o_ref, lse_ref, _ = oracle.attention(q, k, v)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13)
    dout = np.random.default_rng(61).standard_normal(q.shape)
    for a, b in zip(oracle.attention_bwd_ex(q, k, v, lse, dout, window=window),
                    oracle.attention_bwd(q, k, v, lse_ref, dout)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_attention_ex_window_zero_sees_only_itself():
    B, T, H, Hkv, hd = 1, 7, 4, 2, 8
    q, k, v = _qkv(62, B, T, H, Hkv, hd)
    o, lse = oracle.attention_ex(q, k, v, window=0)
    kv = np.repeat(np.arange(Hkv), H // Hkv)
    np.testing.assert_allclose(o, v[:, :, kv, :], rtol=1e-14)
    s = np.einsum("bthd,bthd->bht", q, k[:, :, kv, :]) / math.sqrt(hd)
    np.testing.assert_allclose(lse, s, rtol=1e-13)


def test_attention_ex_groups_equal_repeated_heads():
    """GQA is MHA on K/V heads repeated over each group; the K/V gradients
    are the sums of the repeated heads' gradients (the pinned MHA oracle)."""
    B, T, H, Hkv, hd = 2, 11, 6, 2, 8
    q, k, v = _qkv(63, B, T, H, Hkv, hd)
    rep = np.repeat(np.arange(Hkv), H // Hkv)
    o, lse = oracle.attention_ex(q, k, v)
    o_ref, lse_ref, _ = oracle.attention(q, k[:, :, rep, :], v[:, :, rep, :])
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-14)
    dout = np.random.default_rng(64).standard_normal(q.shape)
    dq, dk, dv = oracle.attention_bwd_ex(q, k, v, lse, dout)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k[:, :, rep, :], v[:, :, rep, :], lse_ref, dout)
    np.testing.assert_allclose(dq, dq_r, rtol=1e-12, atol=1e-13)
    g = H // Hkv
    np.testing.assert_allclose(dk, dk_r.reshape(B, T, Hkv, g, hd).sum(3), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, dv_r.reshape(B, T, Hkv, g, hd).sum(3), rtol=1e-12, atol=1e-13)


def test_attention_ex_window_brute_force():
    """Tiny case against an explicit masked softmax written here."""
    B, T, H, Hkv, hd, W = 1, 10, 4, 2, 5, 3
    q, k, v = _qkv(65, B, T, H, Hkv, hd)
    o, lse = oracle.attention_ex(q, k, v, window=W)
    for h in range(H):
        hk = h // (H // Hkv)
        for t in range(T):
            js = [j for j in range(T) if t - W <= j <= t]
            s = np.array([q[0, t, h] @ k[0, j, hk] for j in js]) / math.sqrt(hd)
            p = np.exp(s - s.max())
            p /= p.sum()
            np.testing.assert_allclose(o[0, t, h], p @ v[0, js, hk], rtol=1e-12)
            np.testing.assert_allclose(lse[0, h, t], s.max() + math.log(np.exp(s - s.max()).sum()),
                                       rtol=1e-13)


def test_attention_ex_backward_finite_differences():
    B, T, H, Hkv, hd, W = 1, 6, 4, 2, 3, 2
    q, k, v = _qkv(66, B, T, H, Hkv, hd)
    R = np.random.default_rng(67).standard_normal(q.shape)
    loss = lambda q_, k_, v_: float((oracle.attention_ex(q_, k_, v_, window=W)[0] * R).sum())
    o, lse = oracle.attention_ex(q, k, v, window=W)
    grads = oracle.attention_bwd_ex(q, k, v, lse, R, window=W)
    rng = np.random.default_rng(68)
    eps = 1e-6
    for which, x in enumerate((q, k, v)):
        for _ in range(6):
            idx = tuple(rng.integers(0, n) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grads[which][idx]) < 1e-6 * max(1.0, abs(fd)), (which, idx)


# ------------------------------------------------------------------ AdamW (embeddings, lm_head)
ADAM = dict(lr=0.01, b1=0.9, b2=0.95, eps=1e-8)


def test_adamw_first_step_is_a_normalised_sign_step():
    """Step 1 with no decay: bias correction makes m-hat = g and v-hat = g^2
    exactly, so each weight moves by lr * g / (|g| + eps); g = 0 stays put."""
    rng = np.random.default_rng(30)
    W, g = rng.standard_normal(500), rng.standard_normal(500)
    g[::7] = 0.0
    z = np.zeros(500)
    W1, m1, v1 = oracle.adamw_update(W, z, z, g, wd=0.0, t=1, **ADAM)
    np.testing.assert_allclose(W - W1, ADAM["lr"] * g / (np.abs(g) + ADAM["eps"]), rtol=1e-12, atol=1e-18)
    assert np.all(W1[::7] == W[::7])


def test_adamw_constant_gradient_moves_linearly():
    """With the same g every step the bias-corrected moments stay g and g^2,
    so after t steps W = W0 - t * lr * g / (|g| + eps) (no decay)."""
    rng = np.random.default_rng(31)
    W0, g = rng.standard_normal(300), rng.standard_normal(300)
    W, m, v = W0, np.zeros(300), np.zeros(300)
    for t in range(1, 8):
        W, m, v = oracle.adamw_update(W, m, v, g, wd=0.0, t=t, **ADAM)
        np.testing.assert_allclose(W0 - W, t * ADAM["lr"] * g / (np.abs(g) + ADAM["eps"]), rtol=1e-10)


def test_adamw_decay_is_decoupled():
    """Zero gradient: the moments stay zero and only the decoupled decay acts,
    W_t = W0 (1 - lr wd)^t (a decay folded into g would move m and v)."""
    rng = np.random.default_rng(32)
    W0 = rng.standard_normal(200)
    W, m, v = W0, np.zeros(200), np.zeros(200)
    wd = 0.1
    for t in range(1, 5):
        W, m, v = oracle.adamw_update(W, m, v, np.zeros(200), wd=wd, t=t, **ADAM)
        assert np.all(m == 0) and np.all(v == 0)
        np.testing.assert_allclose(W, W0 * (1 - ADAM["lr"] * wd) ** t, rtol=1e-13)


def test_adamw_moments_after_two_steps():
    rng = np.random.default_rng(33)
    g1, g2 = rng.standard_normal(100), rng.standard_normal(100)
    z = np.zeros(100)
    b1, b2 = ADAM["b1"], ADAM["b2"]
    W1, m1, v1 = oracle.adamw_update(z, z, z, g1, wd=0.0, t=1, **ADAM)
    W2, m2, v2 = oracle.adamw_update(W1, m1, v1, g2, wd=0.0, t=2, **ADAM)
    np.testing.assert_allclose(m2, (1 - b1) * (b1 * g1 + g2), rtol=1e-13)
    np.testing.assert_allclose(v2, (1 - b2) * (b2 * g1 ** 2 + g2 ** 2), rtol=1e-13)
    mhat, vhat = m2 / (1 - b1 ** 2), v2 / (1 - b2 ** 2)
    np.testing.assert_allclose(W1 - W2, ADAM["lr"] * mhat / (np.sqrt(vhat) + ADAM["eps"]), rtol=1e-10)


def test_adamw_is_invariant_to_gradient_scale_and_odd_in_its_sign():
    """With eps = 0 the update depends on g only through its direction per
    element: scaling every gradient by c > 0 changes nothing, and flipping the
    sign of g flips the step (both fail if the square root or a moment is
    misplaced)."""
    rng = np.random.default_rng(34)
    W0 = rng.standard_normal(120)
    gs = [rng.standard_normal(120) for _ in range(3)]
    hp = dict(ADAM, eps=0.0)

    def run(scale):
        W, m, v = W0, np.zeros(120), np.zeros(120)
        for t, g in enumerate(gs, 1):
            W, m, v = oracle.adamw_update(W, m, v, scale * g, wd=0.0, t=t, **hp)
        return W

    base = run(1.0)
    np.testing.assert_allclose(run(37.5), base, rtol=1e-12)
    np.testing.assert_allclose(W0 - run(-2.0), -(W0 - base), rtol=1e-10)


# ------------------------------------------------------------------ forward composition
def _rms(x):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-6)


def _logits(depth, P, tok, tgt):
    _, _, z = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, grads=False, want_logits=True)
    return z


def test_forward_attention_branch_closed_form():
    """q = k = 0 (zero Wq, Wk) makes attention uniform over the causal prefix
    and a zero W_up silences the MLP, so one layer reduces to
    z = rms(x0 + cummean(rms(x0) Wv^T) Wo^T) Wlm^T with x0 = E[tok]."""
    depth, T = 1, 7
    P = inputs.random_params(depth, seed=20, vocab=V_SMALL, head_std=0.5)
    P[1][:] = 0
    P[2][:] = 0
    P[5][:] = 0
    tok, tgt = inputs.token_batch(21, 1, T, vocab=V_SMALL)
    x0 = P[0][tok[0]].astype(np.float64)
    v = _rms(x0) @ P[3].astype(np.float64).T
    o = np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None]
    x1 = x0 + o @ P[4].astype(np.float64).T
    z = _rms(x1) @ P[-1].astype(np.float64).T
    np.testing.assert_allclose(_logits(depth, P, tok, tgt), z, rtol=1e-11, atol=1e-12)


def test_forward_mlp_branch_closed_form():
    """A zero Wo silences attention, so one layer is
    z = rms(x0 + relu(rms(x0) Wup^T)^2 Wdown^T) Wlm^T."""
    depth, T = 1, 5
    P = inputs.random_params(depth, seed=22, vocab=V_SMALL, head_std=0.5)
    P[4][:] = 0
    tok, tgt = inputs.token_batch(23, 1, T, vocab=V_SMALL)
    x0 = P[0][tok[0]].astype(np.float64)
    a = np.maximum(_rms(x0) @ P[5].astype(np.float64).T, 0) ** 2
    x1 = x0 + a @ P[6].astype(np.float64).T
    z = _rms(x1) @ P[-1].astype(np.float64).T
    np.testing.assert_allclose(_logits(depth, P, tok, tgt), z, rtol=1e-11, atol=1e-12)


def test_forward_two_positions_brute_force():
    """T = 2, one head, MLP off: the second position mixes two values with
    weights softmax(q1.k0, q1.k1)/sqrt(hd) after RoPE (positions 0, 1) and
    QK-norm; written out here from the definitions."""
    depth = 1
    P = inputs.random_params(depth, seed=24, vocab=V_SMALL, head_std=0.5)
    P[5][:] = 0
    tok, tgt = inputs.token_batch(25, 1, 2, vocab=V_SMALL)
    Wq, Wk, Wv, Wo = (P[i].astype(np.float64) for i in (1, 2, 3, 4))
    x0 = P[0][tok[0]].astype(np.float64)
    h = _rms(x0)
    q, k, v = h @ Wq.T, h @ Wk.T, h @ Wv.T

    def rot(u, pos):  # pairs (i, i + 32) of a 64-wide head, theta_i = pos * 10000^(-i/32)
        th = pos * 10000.0 ** (-np.arange(32) / 32.0)
        a, b = u[:32], u[32:]
        return np.concatenate([a * np.cos(th) - b * np.sin(th), a * np.sin(th) + b * np.cos(th)])

    qh = [_rms(rot(q[t], t)) for t in range(2)]
    kh = [_rms(rot(k[t], t)) for t in range(2)]
    s = np.array([qh[1] @ kh[0], qh[1] @ kh[1]]) / 8.0
    w = np.exp(s - s.max())
    w /= w.sum()
    o = np.stack([v[0], w[0] * v[0] + w[1] * v[1]])
    z = _rms(x0 + o @ Wo.T) @ P[-1].astype(np.float64).T
    np.testing.assert_allclose(_logits(depth, P, tok, tgt), z, rtol=1e-11, atol=1e-12)


def test_qk_norm_makes_loss_invariant_to_q_k_scale():
    depth, T = 2, 9
    P = inputs.random_params(depth, seed=26, vocab=V_SMALL, head_std=0.5)
    tok, tgt = inputs.token_batch(27, 1, T, vocab=V_SMALL)
    # Large q and k make the eps inside the norm negligible (relative 1e-10).
    for i in (1, 2, 7, 8):
        P[i] *= 100.0
    l0, _, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, grads=False)
    Q = [p.copy() for p in P]
    Q[1] *= 4.0  # wq of layer 0
    Q[8] *= 0.5  # wk of layer 1
    l1, _, _ = oracle.gpt_fwd_bwd(depth, Q, tok, tgt, vocab=V_SMALL, grads=False)
    assert abs(l0 - l1) < 1e-9
    Q[3] *= 4.0  # wv is not normalised
    l2, _, _ = oracle.gpt_fwd_bwd(depth, Q, tok, tgt, vocab=V_SMALL, grads=False)
    assert abs(l0 - l2) > 1e-4


def test_head_and_hidden_permutations_leave_loss_unchanged():
    depth, T = 4, 6  # d = 256: two heads of 128
    P = inputs.random_params(depth, seed=28, vocab=V_SMALL, head_std=0.5)
    tok, tgt = inputs.token_batch(29, 1, T, vocab=V_SMALL)
    l0, _, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, grads=False)
    Q = [p.copy() for p in P]
    perm_heads = np.concatenate([np.arange(128, 256), np.arange(0, 128)])
    perm_hidden = np.random.default_rng(30).permutation(1024)
    for l in range(depth):
        b = 1 + 6 * l
        for j in range(3):
            Q[b + j] = Q[b + j][perm_heads]
        Q[b + 3] = Q[b + 3][:, perm_heads]
        Q[b + 4] = Q[b + 4][perm_hidden]
        Q[b + 5] = Q[b + 5][:, perm_hidden]
    l1, _, _ = oracle.gpt_fwd_bwd(depth, Q, tok, tgt, vocab=V_SMALL, grads=False)
    assert abs(l0 - l1) < 1e-10
    # Mixing a head's halves is not a symmetry: RoPE pairs i with i + 64.
    R = [p.copy() for p in P]
    swap = np.concatenate([np.arange(64, 128), np.arange(0, 64), np.arange(128, 256)])
    R[1], R[2] = R[1][swap], R[2][swap]
    l2, _, _ = oracle.gpt_fwd_bwd(depth, R, tok, tgt, vocab=V_SMALL, grads=False)
    assert abs(l0 - l2) > 1e-6


# ------------------------------------------------ model with grouped KV heads and windows
# Guide, section "1. Modelo GPT": fewer KV heads (GQA) and a short/long window
# alternating across layers ("SSSL"); the window is the attention call's
# window_size.  Reading: query head h reads KV head h // (H / Hkv); a window w
# lets query t see keys t - w .. t.

def _repeat_kv(P, depth, H, Hkv):
    """MHA parameters equivalent to grouped ones: KV head g's rows repeated
    for each query head h with h // (H / Hkv) == g."""
    Q = [p.copy() for p in P]
    group = H // Hkv
    for l in range(depth):
        for j in (1, 2):
            w = P[1 + 6 * l + j]
            Q[1 + 6 * l + j] = np.repeat(w.reshape(Hkv, 128, -1), group, axis=0).reshape(H * 128, -1)
    return Q


def test_model_grouped_kv_equals_repeated_kv_heads():
    """depth 8: four query heads on two KV heads.  The grouped model equals the
    multi-head model whose wk / wv repeat each KV head for its group, in loss,
    logits and every gradient; the KV gradient is the sum over the group.  A
    mapping h % Hkv instead of h // group fails here."""
    depth, T, H, Hkv = 8, 6, 4, 2
    P = inputs.random_params(depth, seed=40, vocab=V_SMALL, head_std=0.5, n_kv_head=Hkv)
    tok, tgt = inputs.token_batch(41, 2, T, vocab=V_SMALL)
    lg, Gg, zg = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, want_logits=True,
                                    n_kv_head=Hkv)
    Q = _repeat_kv(P, depth, H, Hkv)
    lm, Gm, zm = oracle.gpt_fwd_bwd(depth, Q, tok, tgt, vocab=V_SMALL, want_logits=True)
    assert abs(lg - lm) < 1e-12
    np.testing.assert_allclose(zg, zm, rtol=0, atol=1e-11)
    for i, (gg, gm) in enumerate(zip(Gg, Gm)):
        l, j = (i - 1) // 6, (i - 1) % 6
        if 1 <= i <= 6 * depth and j in (1, 2):
            gm = gm.reshape(Hkv, H // Hkv, 128, -1).sum(axis=1).reshape(gg.shape)
        np.testing.assert_allclose(gg, gm, rtol=1e-9, atol=1e-12 * np.abs(gm).max())
    # The other mapping (h % Hkv) is a different model.
    R = [p.copy() for p in Q]
    for l in range(depth):
        for j in (1, 2):
            w = P[1 + 6 * l + j].reshape(Hkv, 128, -1)
            R[1 + 6 * l + j] = np.concatenate([w] * (H // Hkv), axis=0).reshape(H * 128, -1)
    lr, _, _ = oracle.gpt_fwd_bwd(depth, R, tok, tgt, vocab=V_SMALL, grads=False)
    assert abs(lg - lr) > 1e-6


def test_model_window_covering_the_row_is_full_causal():
    depth, T = 4, 9
    P = inputs.random_params(depth, seed=42, vocab=V_SMALL, head_std=0.5, n_kv_head=1)
    tok, tgt = inputs.token_batch(43, 1, T, vocab=V_SMALL)
    l0, G0, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, n_kv_head=1)
    l1, G1, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, n_kv_head=1,
                                   window=[T - 1, -1, T + 5, T - 1])
    assert abs(l0 - l1) < 1e-12  # the loss is an OpenMP reduction: order not fixed
    assert all(np.array_equal(a, b) for a, b in zip(G0, G1))
    l2, _, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, n_kv_head=1,
                                  window=[T - 2, -1, -1, -1], grads=False)
    assert abs(l2 - l0) > 1e-6  # the last query loses its first key


def test_model_window_zero_makes_positions_independent():
    """With w = 0 every query sees only its own key, so attention returns v and
    position t's logits depend on token t alone: they equal those of a row of
    length 1 holding that token (RoPE and the scores drop out)."""
    depth, T = 4, 7
    P = inputs.random_params(depth, seed=44, vocab=V_SMALL, head_std=0.5, n_kv_head=1)
    tok, tgt = inputs.token_batch(45, 1, T, vocab=V_SMALL)
    _, _, z = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, grads=False, want_logits=True,
                                 n_kv_head=1, window=[0] * depth)
    _, _, z1 = oracle.gpt_fwd_bwd(depth, P, tok.reshape(T, 1), tgt.reshape(T, 1), vocab=V_SMALL,
                                  grads=False, want_logits=True, n_kv_head=1)
    np.testing.assert_allclose(z, z1, rtol=0, atol=1e-12)


def test_model_window_receptive_field_is_depth_times_window():
    """Windows w in all L layers: position t reads tokens t - L*w .. t.  A token
    change at p leaves logits beyond p + L*w bit-identical and changes the
    logits at p + L*w (an off-by-one in the window's edge fails one side).  A
    full-causal layer among them reaches every later position."""
    depth, T, w, p = 4, 16, 2, 1
    P = inputs.random_params(depth, seed=46, vocab=V_SMALL, head_std=0.5, n_kv_head=2)
    tok, tgt = inputs.token_batch(47, 1, T, vocab=V_SMALL)
    tok2 = tok.copy()
    tok2[0, p] = (tok2[0, p] + 1) % V_SMALL

    def z(t, window):
        return oracle.gpt_fwd_bwd(depth, P, t, tgt, vocab=V_SMALL, grads=False, want_logits=True,
                                  n_kv_head=2, window=window)[2]

    za, zb = z(tok, [w] * depth), z(tok2, [w] * depth)
    edge = p + depth * w
    assert np.array_equal(za[:p], zb[:p])
    assert np.array_equal(za[edge + 1:], zb[edge + 1:])
    assert not np.allclose(za[edge], zb[edge], rtol=0, atol=1e-9)
    pattern = oracle.window_pattern("SSSL", depth, w)
    assert pattern == [w, w, w, -1]
    zc, zd = z(tok, pattern), z(tok2, pattern)
    assert all(not np.allclose(zc[t], zd[t], rtol=0, atol=1e-9) for t in range(p, T))


def test_model_grouped_windowed_gradients_central_finite_differences():
    """Central differences through a depth-4 model with one KV head for two
    query heads and windows (2, full, 0, 5) at T = 8, every tensor."""
    depth, T, window = 4, 8, [2, -1, 0, 5]
    P = inputs.random_params(depth, seed=48, vocab=V_SMALL, head_std=0.5, bf16_exact=False,
                             n_kv_head=1)
    tok, tgt = inputs.token_batch(49, 1, T, vocab=V_SMALL)
    _, G, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, n_kv_head=1, window=window)
    rng = np.random.default_rng(50)
    h = 2.0 ** -12
    for ti, (p, g) in enumerate(zip(P, G)):
        scale = np.abs(g).max()
        # At w = 0 a query sees only its own key: q and k drop out, so wq and
        # wk of that layer get exactly zero gradient; every other tensor not.
        dead = 1 <= ti <= 6 * depth and window[(ti - 1) // 6] == 0 and (ti - 1) % 6 in (0, 1)
        assert (scale == 0) == dead, ti
        scale = scale if scale > 0 else 1e-6
        picks = [np.unravel_index(np.argmax(np.abs(g)), g.shape)]
        picks += [tuple(rng.integers(0, s) for s in g.shape) for _ in range(2)]
        if ti == 0:
            picks = [(int(tok[0, j]), int(rng.integers(0, p.shape[1]))) for j in range(2)]
        for idx in picks:
            Pp = [q.copy() for q in P]
            Pm = [q.copy() for q in P]
            Pp[ti][idx] += np.float32(h)
            Pm[ti][idx] -= np.float32(h)
            lp = oracle.gpt_fwd_bwd(depth, Pp, tok, tgt, vocab=V_SMALL, grads=False, n_kv_head=1,
                                    window=window)[0]
            lm = oracle.gpt_fwd_bwd(depth, Pm, tok, tgt, vocab=V_SMALL, grads=False, n_kv_head=1,
                                    window=window)[0]
            fd = (lp - lm) / (float(Pp[ti][idx]) - float(Pm[ti][idx]))
            assert abs(fd - g[idx]) <= 2e-5 * scale + 1e-9, (ti, idx, fd, g[idx], scale)


def test_model_grouped_kv_shapes_and_bad_counts():
    s = oracle.dims(8, V_SMALL, n_kv_head=2)
    assert (s["n_head"], s["n_kv_head"]) == (4, 2)
    assert oracle.param_shapes(8, V_SMALL, 2)[2] == (256, 512)
    assert oracle.param_numel(8, 2, V_SMALL, n_kv_head=2) == 256 * 512
    assert oracle.param_shapes(8, V_SMALL, 2) == inputs.param_shapes(8, V_SMALL, 2)
    for bad in (3, 5, 8):
        with pytest.raises(ValueError):
            oracle.dims(8, V_SMALL, n_kv_head=bad)


# ------------------------------------------------------------------ FP8 (E4M3)
# The OCP 8-bit format E4M3, built here from its definition: 1 sign, 4
# exponent bits (bias 7), 3 mantissa bits; exponent field 0 is subnormal
# (m/8 * 2^-6); the code S.1111.111 is NaN, so the largest finite is
# 1.75 * 2^8 = 448; no infinities.

def _e4m3_table():
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # NaN
            vals.append(m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(sorted(vals))  # 127 non-negative finite values


def _e4m3_nearest(x, table):
    """Brute force: the table entry nearest |x|, ties to the even code, then
    the sign; saturating at 448."""
    out = np.empty_like(x)
    codes = np.arange(len(table))  # sorted order == code order for non-negatives
    for i, v in enumerate(x):
        a = min(abs(v), 448.0)
        dist = np.abs(table - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:  # a tie: the even code, i.e. the even mantissa
            best = best[codes[best] % 2 == 0]
        out[i] = math.copysign(table[best[0]], v)
    return out


def test_e4m3_table_has_the_format_landmarks():
    t = _e4m3_table()
    assert len(t) == 127 and t[0] == 0 and t[-1] == 448.0
    assert t[1] == 2.0 ** -9 and 2.0 ** -6 in t and 240.0 in t and 480.0 not in t


def test_e4m3_round_is_the_nearest_value_ties_to_even():
    t = _e4m3_table()
    rng = np.random.default_rng(60)
    x = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.uniform(-4, 3, 3000),  # every binade
        (t[1:] + t[:-1]) / 2,                                           # every midpoint
        -(t[1:] + t[:-1]) / 2,
        t, -t, [449.0, 463.9, 464.0, 1e6, -1e30],                       # saturation
    ])
    np.testing.assert_array_equal(oracle.e4m3_round(x), _e4m3_nearest(x, t))


def test_e4m3_round_special_values():
    r = oracle.e4m3_round([np.inf, -np.inf, np.nan, 0.0, -0.0])
    assert r[0] == 448 and r[1] == -448 and np.isnan(r[2]) and r[3] == 0
    assert math.copysign(1, r[4]) == -1


def test_fp8_scale_is_448_over_amax_in_fp32():
    x = np.array([0.3, -1.7, 0.01])
    assert oracle.fp8_scale(x) == np.float32(448.0) / np.float32(1.7)
    # an activation's amax is that of its bf16 value (1.7 -> 1.703125)
    assert oracle.fp8_scale(x, activation=True) == np.float32(448.0) / np.float32(1.703125)
    assert oracle.fp8_scale(np.zeros(5)) == 1.0


def test_fp8_matmul_brute_force():
    """Per-tensor scaling and E4M3 rounding written here with the table:
    y = (Q(x) Q(w)^T) / (s_x s_w), Q(t) = e4m3(v * s_t) with v the value a
    kernel holds: bf16 for the activation x, fp32 for the weight w."""
    t = _e4m3_table()
    rng = np.random.default_rng(61)
    x = rng.standard_normal((5, 24)) * 3.0
    w = rng.standard_normal((7, 24)) * 0.02
    qx, sx = _quant_table(x, t, act=True)
    qw, sw = _quant_table(w, t)
    ref = qx @ qw.T / (sx * sw)
    np.testing.assert_allclose(oracle.fp8_matmul_nt(x, w), ref, rtol=1e-12, atol=1e-15)
    # Scaling alone is exact up to fp32 rounding of the operands.
    np.testing.assert_allclose(oracle.fp8_matmul_nt(x, w, "scale"), x @ w.T, rtol=1e-5,
                               atol=1e-6 * np.abs(x @ w.T).max())
    # The error is the format's resolution: rounding to 3 mantissa bits leaves
    # an RMS relative error near 2^-3 / sqrt(12) / 1.44 = 2.5% per operand,
    # about 3.5% for the product of two (Gaussian operands, K = 256).
    g = np.random.default_rng(67)
    xg, wg = g.standard_normal((64, 256)), g.standard_normal((128, 256))
    exact = xg @ wg.T
    rel = np.linalg.norm(oracle.fp8_matmul_nt(xg, wg) - exact) / np.linalg.norm(exact)
    assert 0.025 < rel < 0.05, rel


def test_fp8_matmul_is_invariant_to_power_of_two_scaling():
    """s absorbs a factor 2^j exactly, so the quantised codes do not move."""
    rng = np.random.default_rng(62)
    x = rng.standard_normal((6, 32))
    w = rng.standard_normal((5, 32))
    y = oracle.fp8_matmul_nt(x, w)
    np.testing.assert_array_equal(oracle.fp8_matmul_nt(x * 8.0, w / 32.0), y / 4.0)


def test_fp8_model_scaling_alone_is_the_exact_model():
    """With scaling but no rounding, the FP8 plumbing (which operand is scaled
    by which factor, the fused q|k|v tensor) must give back the exact model
    up to fp32 rounding of the GEMM operands."""
    depth, T = 4, 8
    P = inputs.random_params(depth, seed=63, vocab=V_SMALL, head_std=0.5, n_kv_head=1)
    tok, tgt = inputs.token_batch(64, 2, T, vocab=V_SMALL)
    win = [3, -1, 0, 5]
    l0, G0, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, n_kv_head=1, window=win)
    l1, G1, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, n_kv_head=1, window=win,
                                   fp8="scale")
    assert abs(l1 - l0) < 1e-6 * abs(l0)
    for i, (a, b) in enumerate(zip(G0, G1)):
        tol = 1e-5 * max(np.abs(a).max(), 1e-12)
        np.testing.assert_allclose(b, a, rtol=0, atol=tol, err_msg=str(i))


def test_fp8_model_e4m3_is_close_to_the_exact_model():
    """E4M3 operands: the loss moves by well under 1% and each gradient by the
    few-percent-per-GEMM error compounded along its path (under 30% here,
    depth 2), yet visibly; lm_head's own product stays exact, so its
    gradient is among the closest."""
    depth, T = 2, 16
    P = inputs.random_params(depth, seed=65, vocab=V_SMALL, head_std=0.05)
    tok, tgt = inputs.token_batch(66, 2, T, vocab=V_SMALL)
    l0, G0, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL)
    l1, G1, _ = oracle.gpt_fwd_bwd(depth, P, tok, tgt, vocab=V_SMALL, fp8="e4m3")
    assert 1e-5 < abs(l1 - l0) < 1e-2 * abs(l0)
    rel = [np.linalg.norm(b - a) / np.linalg.norm(a) for a, b in zip(G0, G1)]
    assert all(1e-3 < r < 0.3 for r in rel), rel
    assert rel[-1] < 0.15 and rel[-1] <= np.median(rel)


def _quant_table(a, t, act=False):
    """Q(a) and s written here: s = 448 / amax in fp32, codes from the table;
    an activation is first rounded to bf16 (the value a kernel holds)."""
    a32 = np.asarray(a, dtype=np.float32)
    if act:
        a32 = inputs.round_to_bf16(a32)
    amax = np.abs(a32).max()
    s = np.float32(448.0) / amax if amax > 0 else np.float32(1.0)
    y = (a32 * s).astype(np.float64)  # the fp32 product
    return _e4m3_nearest(y.ravel(), t).reshape(a32.shape), float(s)


def test_fp8_rounding_decision_is_taken_on_the_fp32_product():
    """Values whose fp32 product x * s lands exactly on an E4M3 tie although
    the exact product does not: the code follows the fp32 product (ties to
    even), as a kernel's would."""
    t = _e4m3_table()
    s = np.float32(448.0) / np.float32(3.3)  # amax 3.3 sets s
    picked = []
    for tie in ((t[1:] + t[:-1]) / 2)[20:120]:
        c = np.float32(tie / float(s))
        for x in (np.nextafter(c, np.float32(0)), c, np.nextafter(c, np.float32(10))):
            exact = float(x) * float(s)
            if float(np.float32(x) * s) == tie and exact != tie:
                picked.append(float(x))
    assert len(picked) >= 10
    # The values go in as a weight (quantised from fp32); the activation is the
    # identity, whose codes are exact (448 at s = 448), so y[j] = Q(w)_j / s_w.
    w = np.array([[3.3] + picked])
    qw, sw = _quant_table(w, t)
    y = oracle.fp8_matmul_nt(np.eye(w.shape[1]), w)[:, 0]
    np.testing.assert_allclose(y, qw[0] / sw, rtol=1e-12, atol=0)  # codes 1/8 apart


def test_fp8_model_mlp_gradients_brute_force():
    """depth 1 with wo = 0: attention adds nothing, so the MLP sees the
    embedding and everything its weight gradients need is computed here on
    quantised operands (Q(t) = e4m3(v s_t), s_t = 448 / amax, v = bf16(t)
    for activations and gradients, fp32(t) for the weights):
      u = Q(h) Q(wup)^T / ss, a = relu(u)^2, m = Q(a) Q(wdown)^T / ss,
      x_f = x + m, loss through the final RMSNorm and the exact lm_head;
      dW_down = Q(dx_f)^T Q(a) / ss,  da = Q(dx_f) Q(wdown) / ss,
      du = 2 relu(u) da,  dW_up = Q(du)^T Q(h) / ss.
    This covers a forward, an input-gradient and two weight-gradient GEMMs."""
    V, T = V_SMALL, 6
    t = _e4m3_table()
    P = inputs.random_params(1, seed=68, vocab=V, head_std=0.5)
    P[4] = np.zeros_like(P[4])  # wo
    tok, tgt = inputs.token_batch(70, 2, T, vocab=V)
    _, G, _ = oracle.gpt_fwd_bwd(1, P, tok, tgt, vocab=V, fp8="e4m3")
    N = tok.size

    def qmm(a, b, a_act=True, b_act=True):  # a b^T on quantised operands
        qa, sa = _quant_table(a, t, a_act)
        qb, sb = _quant_table(b, t, b_act)
        return qa @ qb.T / (sa * sb)

    def rms_fwd_bwd(x, dy=None):
        r = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6)
        if dy is None:
            return x * r
        return r * dy - (r ** 3 / x.shape[1]) * x * np.sum(dy * x, axis=1, keepdims=True)

    x = P[0][tok.ravel()].astype(np.float64)
    h = rms_fwd_bwd(x)
    u = qmm(h, P[5], b_act=False)
    a = np.maximum(u, 0.0) ** 2
    xf = x + qmm(a, P[6], b_act=False)
    lm = P[-1].astype(np.float64)
    z = rms_fwd_bwd(xf) @ lm.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    p[np.arange(N), tgt.ravel()] -= 1.0
    dxf = rms_fwd_bwd(xf, (p / N) @ lm)
    dwdown = qmm(dxf.T, a.T)          # Q(dx_f)^T Q(a)
    da = qmm(dxf, P[6].T.copy(), b_act=False)  # Q(dx_f) Q(wdown)
    du = 2.0 * np.maximum(u, 0.0) * da
    dwup = qmm(du.T, h.T)
    for got, ref in ((G[6], dwdown), (G[5], dwup)):
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    assert not np.any(G[1]) and not np.any(G[2]) and not np.any(G[3])  # wq wk wv: wo = 0
