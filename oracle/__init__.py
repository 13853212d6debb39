"""ctypes binding of the CPU oracle.

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline and reference legs may import this package; the product
package never does.  Arrays in and out are numpy float64 (float32 for
parameters, int32 for token ids), C-contiguous.
"""
import ctypes
import os

import numpy as np

from .build_oracle import build as _build

_lib = None

NS_COEFFS = (3.4445, -4.7750, 2.0315)
NS_STEPS = 5
NS_EPS = 1e-7
NORM_EPS = 1e-6


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        i64p = ctypes.POINTER(ctypes.c_int64)
        dp = ctypes.POINTER(ctypes.c_double)
        L.oc_dims.argtypes = [ctypes.c_int, ctypes.c_int, i64p]
        L.oc_param_numel.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.oc_param_numel.restype = ctypes.c_int64
        L.oc_splitmix64.argtypes = [ctypes.c_uint64]
        L.oc_splitmix64.restype = ctypes.c_uint64
        L.oc_init_params.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int,
                                     ctypes.c_void_p]
        L.oc_rmsnorm.argtypes = [dp, ctypes.c_int64, ctypes.c_int, ctypes.c_double, dp, dp]
        L.oc_rope_row.argtypes = [dp, ctypes.c_int, ctypes.c_int64, ctypes.c_double]
        L.oc_attention.argtypes = [dp, dp, dp] + [ctypes.c_int] * 4 + [dp, dp, dp]
        L.oc_attention_bwd.argtypes = [dp, dp, dp, dp, dp] + [ctypes.c_int] * 4 + [dp, dp, dp]
        L.oc_matmul_nt.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, dp]
        L.oc_gpt_fwd_bwd.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_int, ctypes.c_int, dp,
                                     ctypes.c_void_p, dp]
        L.oc_newton_schulz.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                       ctypes.c_double, dp]
        L.oc_muon_update.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                     ctypes.c_double]
        L.oc_attention_ex.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp]
        L.oc_attention_bwd_ex.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          dp, dp, dp]
        L.oc_dims_ex.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, i64p]
        L.oc_param_numel_ex.argtypes = [ctypes.c_int] * 4
        L.oc_param_numel_ex.restype = ctypes.c_int64
        L.oc_init_params_ex.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                        ctypes.c_int, ctypes.c_void_p]
        L.oc_gpt_fwd_bwd_ex.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int, ctypes.c_int, dp, ctypes.c_void_p, dp]
        L.oc_gpt_fwd_bwd_fp8.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_int, dp, ctypes.c_void_p, dp]
        L.oc_threads.argtypes = [ctypes.c_int]
        L.oc_threads.restype = ctypes.c_int
        L.oc_e4m3_round.argtypes = [ctypes.c_double]
        L.oc_e4m3_round.restype = ctypes.c_double
        L.oc_fp8_scale.argtypes = [dp, ctypes.c_int64, ctypes.c_int]
        L.oc_fp8_scale.restype = ctypes.c_float
        L.oc_fp8_matmul_nt.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int, dp]
        L.oc_adamw_update.argtypes = [dp, dp, dp, dp, ctypes.c_int64, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_double, ctypes.c_int]
        _lib = L
    return _lib


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def dims(depth, vocab=32768, n_kv_head=0):
    """Model shape; n_kv_head <= 0 means one KV head per query head."""
    out = (ctypes.c_int64 * 7)()
    if lib().oc_dims_ex(depth, vocab, n_kv_head, out) != 0:
        raise ValueError("invalid depth/vocab/n_kv_head")
    d, H, hd, F, n_t, n_b, Hkv = list(out)
    return dict(d=d, n_head=H, head_dim=hd, mlp=F, n_tensors=n_t, n_block=n_b, vocab=vocab,
                depth=depth, n_kv_head=Hkv)


def param_shapes(depth, vocab=32768, n_kv_head=0):
    s = dims(depth, vocab, n_kv_head)
    d, F, V = s["d"], s["mlp"], vocab
    dkv = s["n_kv_head"] * s["head_dim"]
    shapes = [(V, d)]
    for _ in range(depth):
        shapes += [(d, d), (dkv, d), (dkv, d), (d, d), (F, d), (d, F)]
    shapes.append((V, d))
    return shapes


def window_pattern(pattern, depth, short):
    """Per-layer windows from a short/long pattern string such as "SSSL"
    (guide, section "1. Modelo GPT"): layer l takes pattern[l % len];
    'S' is a left window of `short` keys, 'L' full causal (-1)."""
    if not pattern or any(c not in "SL" for c in pattern):
        raise ValueError("pattern of 'S' and 'L'")
    return [short if pattern[l % len(pattern)] == "S" else -1 for l in range(depth)]


def splitmix64(x):
    return int(lib().oc_splitmix64(ctypes.c_uint64(x & 0xFFFFFFFFFFFFFFFF)))


def init_params(depth, vocab=32768, seed=0, spec_zero=True, n_kv_head=0):
    shapes = param_shapes(depth, vocab, n_kv_head)
    arrs = [np.empty(s, dtype=np.float32) for s in shapes]
    ptrs = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    if lib().oc_init_params_ex(depth, vocab, n_kv_head, seed, 1 if spec_zero else 0, ptrs) != 0:
        raise ValueError("oc_init_params failed")
    return arrs


def rmsnorm(x, eps=NORM_EPS):
    x = _f64(x)
    cols = x.shape[-1]
    rows = x.size // cols
    y = np.empty_like(x)
    r = np.empty(x.shape[:-1], dtype=np.float64)
    assert lib().oc_rmsnorm(_dp(x), rows, cols, eps, _dp(y), _dp(r)) == 0
    return y, r


def rope_row(v, pos, base=10000.0):
    v = _f64(v).copy()
    assert lib().oc_rope_row(_dp(v), v.shape[-1], pos, base) == 0
    return v


def attention(q, k, v, want_probs=False):
    """q, k, v: [B, T, H, hd] -> (o [B, T, H, hd], lse [B, H, T], probs or None)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, hd = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, T), dtype=np.float64)
    probs = np.empty((B, H, T, T), dtype=np.float64) if want_probs else None
    pp = _dp(probs) if want_probs else ctypes.cast(None, ctypes.POINTER(ctypes.c_double))
    assert lib().oc_attention(_dp(q), _dp(k), _dp(v), B, T, H, hd, _dp(o), _dp(lse), pp) == 0
    return o, lse, probs


def attention_bwd(q, k, v, lse, dout):
    """Gradients (dq, dk, dv) of causal attention, layout [B, T, H, hd]."""
    q, k, v, lse, dout = _f64(q), _f64(k), _f64(v), _f64(lse), _f64(dout)
    B, T, H, hd = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    assert lib().oc_attention_bwd(_dp(q), _dp(k), _dp(v), _dp(lse), _dp(dout), B, T, H, hd,
                                  _dp(dq), _dp(dk), _dp(dv)) == 0
    return dq, dk, dv


def attention_ex(q, k, v, window=-1):
    """Causal attention with KV heads k, v: [B, T, Hkv, hd] shared by groups of
    H / Hkv query heads and a left window (-1: none) -> (o, lse)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, hd = q.shape
    Hkv = k.shape[2]
    o = np.empty_like(q)
    lse = np.empty((B, H, T), dtype=np.float64)
    assert lib().oc_attention_ex(_dp(q), _dp(k), _dp(v), B, T, H, Hkv, hd, window, _dp(o),
                                 _dp(lse)) == 0
    return o, lse


def attention_bwd_ex(q, k, v, lse, dout, window=-1):
    """Gradients (dq [B, T, H, hd], dk, dv [B, T, Hkv, hd]) of attention_ex."""
    q, k, v, lse, dout = _f64(q), _f64(k), _f64(v), _f64(lse), _f64(dout)
    B, T, H, hd = q.shape
    Hkv = k.shape[2]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    assert lib().oc_attention_bwd_ex(_dp(q), _dp(k), _dp(v), _dp(lse), _dp(dout), B, T, H, Hkv,
                                     hd, window, _dp(dq), _dp(dk), _dp(dv)) == 0
    return dq, dk, dv


def matmul_nt(x, w):
    x, w = _f64(x), _f64(w)
    rows, k = x.shape
    n = w.shape[0]
    y = np.empty((rows, n), dtype=np.float64)
    assert lib().oc_matmul_nt(_dp(x), _dp(w), rows, n, k, _dp(y)) == 0
    return y


def gpt_fwd_bwd(depth, params, tokens, targets, vocab=32768, grads=True, want_logits=False,
                n_kv_head=0, window=None, fp8=None):
    """Returns (loss, grads list of float64 arrays or None, logits or None).
    n_kv_head: grouped KV heads (<= 0: one per query head); window: None
    (full causal) or one window per layer (negative: full causal); fp8:
    None (exact GEMMs), "e4m3" or "scale" (the block projections' GEMMs on
    scaled operands, rounded to E4M3 or not)."""
    params = [np.ascontiguousarray(p, dtype=np.float32) for p in params]
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    targets = np.ascontiguousarray(targets, dtype=np.int32)
    B, T = tokens.shape
    pptr = (ctypes.c_void_p * len(params))(*[p.ctypes.data for p in params])
    loss = ctypes.c_double(0)
    g = [np.empty(p.shape, dtype=np.float64) for p in params] if grads else None
    gptr = (ctypes.c_void_p * len(params))(*[a.ctypes.data for a in g]) if grads else None
    logits = np.empty((B * T, vocab), dtype=np.float64) if want_logits else None
    lp = _dp(logits) if want_logits else ctypes.cast(None, ctypes.POINTER(ctypes.c_double))
    win = None
    if window is not None:
        win = np.ascontiguousarray(window, dtype=np.int32)
        if win.shape != (depth,):
            raise ValueError("one window per layer")
    wp = win.ctypes.data if win is not None else None
    if fp8 is None:
        rc = lib().oc_gpt_fwd_bwd_ex(depth, vocab, n_kv_head, wp, pptr, tokens.ctypes.data,
                                     targets.ctypes.data, B, T, ctypes.byref(loss), gptr, lp)
    else:
        fmt = {"e4m3": 1, "scale": 0}[fp8]
        rc = lib().oc_gpt_fwd_bwd_fp8(depth, vocab, n_kv_head, wp, fmt, pptr, tokens.ctypes.data,
                                      targets.ctypes.data, B, T, ctypes.byref(loss), gptr, lp)
    if rc == -2:
        raise ValueError("token id out of range")
    if rc != 0:
        raise ValueError("oc_gpt_fwd_bwd failed (%d)" % rc)
    return loss.value, g, logits


def threads(n=0):
    """OpenMP threads of later oracle calls (n > 0 sets them); returns the
    count in effect."""
    return int(lib().oc_threads(n))


def e4m3_round(x):
    """Nearest E4M3 value(s) (ties to even, saturating to 448), elementwise."""
    f = np.vectorize(lambda v: lib().oc_e4m3_round(float(v)), otypes=[np.float64])
    return f(np.asarray(x, dtype=np.float64))


def fp8_scale(x, activation=False):
    """448 / amax of the values x is quantised from (bf16 for an activation)."""
    x = _f64(x)
    return float(lib().oc_fp8_scale(_dp(x), x.size, 1 if activation else 0))


def fp8_matmul_nt(x, w, fmt="e4m3"):
    x, w = _f64(x), _f64(w)
    y = np.empty((x.shape[0], w.shape[0]))
    assert lib().oc_fp8_matmul_nt(_dp(x), _dp(w), x.shape[0], w.shape[0], x.shape[1],
                                  {"e4m3": 1, "scale": 0}[fmt], _dp(y)) == 0
    return y


def newton_schulz(G, steps=NS_STEPS, coeffs=NS_COEFFS, eps=NS_EPS):
    G = _f64(G)
    rows, cols = G.shape
    out = np.empty_like(G)
    a, b, c = coeffs
    assert lib().oc_newton_schulz(_dp(G), rows, cols, steps, a, b, c, eps, _dp(out)) == 0
    return out


def muon_update(W, M, G, lr, mu):
    W, M, G = _f64(W).copy(), _f64(M).copy(), _f64(G)
    rows, cols = W.shape
    assert lib().oc_muon_update(_dp(W), _dp(M), _dp(G), rows, cols, lr, mu) == 0
    return W, M


def adamw_update(W, m, v, g, lr, b1, b2, eps, wd, t):
    """AdamW step t on copies of W, m, v (any shape); returns (W, m, v)."""
    W, m, v, g = _f64(W).copy(), _f64(m).copy(), _f64(v).copy(), _f64(g)
    assert lib().oc_adamw_update(_dp(W), _dp(m), _dp(v), _dp(g), W.size, lr, b1, b2, eps, wd,
                                 t) == 0
    return W, m, v


def param_numel(depth, idx, vocab=32768, n_kv_head=0):
    return int(lib().oc_param_numel_ex(depth, vocab, n_kv_head, idx))
