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


def test_newton_schulz_flops_closed_form():
    """Per iteration, a d x d matrix costs three d^3 products (6 d^3) and a
    d x 4d one X X^T, A A, B X (8 + 2 + 8 = 18 d^3); 4L squares, 2L wide, five
    iterations: 300 L d^3."""
    for depth in (2, 12, 20, 26):
        d = 64 * depth
        assert bench.ns_flops(depth) == 300.0 * depth * d ** 3


def test_training_flops_per_token_at_three_depths():
    """6 N_mm + 6 L d T with N_mm = 12 L d^2 + V d: 0.774, 2.926 and 6.042
    GFLOP per token at depths 12, 20 and 26 (T 2048, V 32768)."""
    for depth, gflop in ((12, 0.774), (20, 2.926), (26, 6.042)):
        assert abs(bench.model_flops_per_token(depth) / 1e9 - gflop) < 5e-4


def test_gemm_byte_model_counts_every_launch_of_the_step():
    """Twelve GEMMs per layer, three for lm_head per 32768-token chunk (two
    chunks of the 65536-token batch) and thirty for Newton-Schulz (five
    iterations of three products on two stacks): 276 at depth 20, with
    231.5 GB of operands and results; one chunk less reads W_lm twice and
    accumulates dW_lm once less (8 B per weight)."""
    total, launches = bench.gemm_algorithmic_bytes_per_step()
    assert launches == 20 * 12 + 2 * 3 + 30 == 276
    assert abs(total / 1e9 - 231.5) < 0.1
    by1, l1 = bench.gemm_algorithmic_bytes_by_class(lm_chunk=bench.B * bench.T)
    assert l1["lmhead"] == 3
    assert total - sum(by1.values()) == bench.V * 64 * bench.DEPTH * 8
    # Doubling the batch doubles every activation term and leaves weights.
    t2, _ = bench.gemm_algorithmic_bytes_per_step(batch=2 * bench.B)
    assert total < t2 < 2 * total


def test_replica_throughput_counts_all_ranks():
    assert bench.replica_tokens_per_s(10, 4, 1000.0) == 10 * bench.B * bench.T * 4


def test_step_times_are_the_gaps_between_marks():
    class Mark:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    marks = [Mark(t) for t in (0.0, 2.0, 5.0, 6.5)]
    assert bench.step_times_ms(marks) == [2.0, 3.0, 1.5]


def test_ns_sweep_flops_match_the_square_and_wide_counts():
    """The Newton-Schulz sweep (64 x 1664^2, 26 x 1664x6656, 26 x 6656x1664, five
    steps): a square n x n matrix costs 6 n^3 per step and a 1 : 4 one 18 m^3
    (m the short side), whichever way it stands: 30.41 TFLOP in all."""
    n = 1664
    assert bench.ns_sweep_flops(((1, n, n),), steps=1) == 6.0 * n ** 3
    assert bench.ns_sweep_flops(((1, n, 4 * n),), steps=1) == 18.0 * n ** 3
    assert bench.ns_sweep_flops(((1, 4 * n, n),), steps=1) == 18.0 * n ** 3
    total = 5 * (64 * 6.0 + 2 * 26 * 18.0) * n ** 3
    assert bench.ns_sweep_flops() == total
    assert abs(total / 1e12 - 30.41) < 0.01


def test_gemm_byte_classes_sum_to_the_step():
    by_class, launches = bench.gemm_algorithmic_bytes_by_class()
    total, n = bench.gemm_algorithmic_bytes_per_step()
    assert sum(by_class.values()) == total and sum(launches.values()) == n
    assert set(by_class) == {"fwd", "dgrad", "wgrad", "lmhead", "ns"}


def test_tensor_peak_at_a_clock():
    """148 SMs x 8192 FLOP per clock: 2.38 PFLOP/s at the 1965 MHz maximum,
    1.82 at 1500 MHz."""
    assert abs(bench.tensor_peak_at(1965.0) - 2382.3) < 0.1
    assert abs(bench.tensor_peak_at(1500.0) - 1818.6) < 0.1
