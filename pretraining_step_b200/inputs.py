"""Seeded synthetic inputs for the pretraining step.

This module is the only code that both the CUDA path's tests and the CPU
oracle consume.  It holds none of the model's arithmetic: it draws token
ids and weight matrices and nothing else.

Token ids: the pages train on web-text shards (ClimbMix / FineWeb-like),
which are not available here; uniform ids over the 32768-entry BPE
vocabulary stand in for them (and a Zipf(1.0) stream for the embedding
scatter stress case).  Each row is a stream of T+1 ids; inputs are ids
[0, T) and next-token targets are ids [1, T+1).

Id i of the stream with key k is  ((splitmix64(k + i) >> 32) * V) >> 32,
which for V = 32768 is the top 15 bits of the SplitMix64 word.
"""
import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_TOKENS = 0x746F6B656E73  # "tokens"


def splitmix64(x):
    """SplitMix64 output for state x (Steele, Lea & Flood 2014), vectorised, uint64."""
    with np.errstate(over="ignore"):
        z = np.asarray(x, dtype=np.uint64) + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def stream_key(seed, stream):
    return splitmix64(np.uint64(seed) ^ splitmix64(np.uint64(stream)))


def uniform_ids(seed, n, vocab, stream=STREAM_TOKENS):
    key = stream_key(seed, stream)
    with np.errstate(over="ignore"):
        w = splitmix64(key + np.arange(n, dtype=np.uint64))
    hi = (w >> np.uint64(32)).astype(np.uint64)
    return ((hi * np.uint64(vocab)) >> np.uint64(32)).astype(np.int32)


def token_batch(seed, B, T, vocab=32768):
    """(inputs [B, T], targets [B, T]) int32, uniform ids, targets = next id."""
    ids = uniform_ids(seed, B * (T + 1), vocab).reshape(B, T + 1)
    return np.ascontiguousarray(ids[:, :T]), np.ascontiguousarray(ids[:, 1:])


def zipf_token_batch(seed, B, T, vocab=32768, s=1.0):
    """Zipf(s)-distributed ids (rank 1 = id 0): the heavy-collision case for the
    embedding scatter.  Drawn by inverse CDF from uniform SplitMix64 words."""
    n = B * (T + 1)
    key = stream_key(seed, STREAM_TOKENS + 1)
    with np.errstate(over="ignore"):
        w = splitmix64(key + np.arange(n, dtype=np.uint64))
    u = (w >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    p = 1.0 / np.arange(1, vocab + 1, dtype=np.float64) ** s
    cdf = np.cumsum(p / p.sum())
    ids = np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1).astype(np.int32)
    ids = ids.reshape(B, T + 1)
    return np.ascontiguousarray(ids[:, :T]), np.ascontiguousarray(ids[:, 1:])


def round_to_bf16(a):
    """Nearest bf16-representable float32 (ties to even), so one array can feed
    a bf16 kernel and a float64 oracle with identical values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).reshape(a.shape)


def param_shapes(depth, vocab=32768, n_kv_head=0):
    """Shapes of the 6*depth + 2 parameter tensors, in interface order:
    wte [V, d]; per layer wq, wk, wv, wo [d, d], wup [4d, d], wdown [d, 4d];
    lm_head [V, d].  d = 64 * depth.  With n_kv_head > 0, wk and wv have
    n_kv_head * head_dim rows (head_dim = min(128, d))."""
    d = 64 * depth
    F = 4 * d
    dkv = n_kv_head * min(128, d) if n_kv_head > 0 else d
    shapes = [(vocab, d)]
    for _ in range(depth):
        shapes += [(d, d), (dkv, d), (dkv, d), (d, d), (F, d), (d, F)]
    shapes.append((vocab, d))
    return shapes


def random_params(depth, seed, vocab=32768, head_std=None, bf16_exact=True, n_kv_head=0):
    """Every tensor drawn N(0, 1/fan_in) (embedding std 1; lm_head std
    head_std, default 1/sqrt(d)), from numpy's PCG64 with the given seed.
    With bf16_exact the values are rounded to bf16 so both sides see the
    same numbers."""
    rng = np.random.default_rng(seed)
    shapes = param_shapes(depth, vocab, n_kv_head)
    d = 64 * depth
    out = []
    for i, (r, c) in enumerate(shapes):
        if i == 0:
            std = 1.0
        elif i == len(shapes) - 1:
            std = head_std if head_std is not None else d ** -0.5
        else:
            std = c ** -0.5
        w = (rng.standard_normal((r, c)) * std).astype(np.float32)
        out.append(round_to_bf16(w) if bf16_exact else w)
    return out


def normal_stack(seed, count, rows, cols, bf16_exact=True):
    """count x [rows, cols] N(0, 1) matrices (Newton-Schulz sweep inputs)."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((count, rows, cols), dtype=np.float32)
    return round_to_bf16(w) if bf16_exact else w


def bf16_normal(seed, shape, std=1.0):
    rng = np.random.default_rng(seed)
    return round_to_bf16((rng.standard_normal(shape) * std).astype(np.float32))
