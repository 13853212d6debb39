"""Host-side arithmetic of bench.py (no GPU): the FLOP count of the model
variants reduces to the headline count, and its window term follows the
(query, key) pairs a causal window leaves."""
import bench


def test_variant_flops_reduce_to_the_headline_count():
    base = bench.model_flops_per_token()
    assert bench.step_flops_per_token(bench.DEPTH, bench.T, bench.V) == base
    assert bench.step_flops_per_token(bench.DEPTH, bench.T, bench.V, 10, [-1] * 20) == base
    assert bench.step_flops_per_token(bench.DEPTH, bench.T, bench.V, 0, [5000] * 20) == base


def test_grouped_kv_heads_shrink_only_wk_and_wv():
    d, L = 64 * bench.DEPTH, bench.DEPTH
    full = bench.step_flops_per_token(L, bench.T, bench.V)
    half = bench.step_flops_per_token(L, bench.T, bench.V, n_kv_head=5)  # dkv = d / 2
    assert full - half == 6.0 * L * 2 * (d // 2) * d


def test_window_term_tracks_the_pairs_a_window_leaves():
    T, depth = 2048, 2
    d = 64 * depth
    for w in (0, 1, 64, 511, 2047):
        pairs = sum(min(t, w) + 1 for t in range(T))      # keys t - w .. t of each query
        term = (bench.step_flops_per_token(depth, T, 8, 0, [w, w]) -
                bench.step_flops_per_token(depth, T, 8, 0, [0, 0]))
        band = term / (2 * 12.0 * d) * T                   # the convention's pair count, minus w = 0
        assert abs(band - (pairs - T)) <= max(1.0, 0.01 * pairs), (w, band, pairs - T)
