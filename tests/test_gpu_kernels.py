"""Kernel-level parity of the CUDA path (through the C ABI) with the oracle.

Inputs come from the seeded generators (bf16-representable, so both sides
see identical numbers); expected values from oracle/ only.
Tolerances: bf16 outputs carry one bf16 rounding (relative 2^-9), so a
relative Frobenius error of 5e-3 bounds them; fp32 outputs accumulate in
fp32 over K <= 1280 products (relative ~1e-6), bound 2e-5.
"""
import numpy as np
import pytest

import oracle
from pretraining_step_b200 import binding as nc
from pretraining_step_b200 import inputs

from gpu_util import dev_bf16, dev_f32, host, rel_fro, torch

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ GEMM
@pytest.mark.parametrize("a_k,b_k", [(1, 1), (1, 0), (0, 1), (0, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 296, 136), (256, 128, 512),
                                   (384, 384, 200), (64, 1280, 1280),
                                   # CTA-pair tiles (256 x 256): ragged M, ragged K
                                   (520, 512, 200), (296, 768, 136), (1024, 1280, 64)])
def test_gemm_layouts(a_k, b_k, M, N, K):
    t = torch()
    A = inputs.bf16_normal(1, (M, K))
    B = inputs.bf16_normal(2, (N, K))
    tA = dev_bf16(A if a_k else A.T)
    tB = dev_bf16(B if b_k else B.T)
    D = t.empty(M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, tA, tB, D, a_kmajor=a_k, b_kmajor=b_k)
    t.cuda.synchronize()
    ref = oracle.matmul_nt(A, B)
    assert rel_fro(host(D), ref) < 5e-3


@pytest.mark.parametrize("a_k,b_k", [(1, 1), (0, 0)])
def test_gemm_f32_store_and_alpha(a_k, b_k):
    t = torch()
    M, N, K = 256, 512, 320
    A = inputs.bf16_normal(3, (M, K))
    B = inputs.bf16_normal(4, (N, K))
    D = t.empty(M, N, dtype=t.float32, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A if a_k else A.T), dev_bf16(B if b_k else B.T), D,
            a_kmajor=a_k, b_kmajor=b_k, epi=nc.EPI_STORE_F32, alpha=0.5)
    t.cuda.synchronize()
    assert rel_fro(host(D), 0.5 * oracle.matmul_nt(A, B)) < 2e-5


@pytest.mark.parametrize("M,N,K", [(300, 384, 256),   # 128-wide tiles on one CTA
                                   (600, 512, 256),   # CTA pairs, ragged M
                                   # more 256 x 256 tiles than CTA pairs: the aux ring
                                   # runs ahead across tile boundaries; ragged M and N
                                   (8200, 1000, 128)])
def test_gemm_residual_relu2_and_backward_epilogues(M, N, K):
    t = torch()
    A = inputs.bf16_normal(5, (M, K))
    B = inputs.bf16_normal(6, (N, K), std=0.1)
    acc = oracle.matmul_nt(A, B)
    R = np.random.default_rng(7).standard_normal((M, N)).astype(np.float32)
    D = t.empty(M, N, dtype=t.float32, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D, epi=nc.EPI_RESID_F32, aux=dev_f32(R))
    t.cuda.synchronize()
    assert rel_fro(host(D), R + acc) < 2e-5
    # ReLU^2
    D2 = t.empty(M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D2, epi=nc.EPI_RELU2)
    t.cuda.synchronize()
    assert rel_fro(host(D2), np.maximum(acc, 0) ** 2) < 5e-3
    # 2 sqrt(a) * acc with a = relu(u)^2 >= 0
    Aux = inputs.round_to_bf16(np.abs(np.random.default_rng(8).standard_normal((M, N)))
                               .astype(np.float32))
    D3 = t.empty(M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D3, epi=nc.EPI_RELU2_BWD, aux=dev_bf16(Aux))
    t.cuda.synchronize()
    assert rel_fro(host(D3), 2 * np.sqrt(Aux.astype(np.float64)) * acc) < 5e-3
    # alpha*acc + beta*aux
    D4 = t.empty(M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D4, epi=nc.EPI_AXPBY_BF16, aux=dev_bf16(Aux),
            alpha=2.0315, beta=-4.775)
    t.cuda.synchronize()
    assert rel_fro(host(D4), 2.0315 * acc - 4.775 * Aux) < 5e-3


def test_gemm_batched_aux_epilogues():
    """Batched (strided) GEMMs with an aux operand, on CTA-pair tiles: the
    alpha*acc + beta*aux form of the Newton-Schulz steps and the fp32 residual."""
    t = torch()
    bt, M, N, K = 3, 520, 512, 192
    A = inputs.bf16_normal(40, (bt, M, K))
    B = inputs.bf16_normal(41, (bt, N, K), std=0.1)
    Aux = inputs.bf16_normal(42, (bt, M, N))
    R = np.random.default_rng(43).standard_normal((bt, M, N)).astype(np.float32)
    D = t.empty(bt, M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D, batch=bt, stride_a=M * K, stride_b=N * K,
            stride_d=M * N, epi=nc.EPI_AXPBY_BF16, aux=dev_bf16(Aux), stride_aux=M * N,
            alpha=-0.5, beta=1.5)
    D2 = t.empty(bt, M, N, dtype=t.float32, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D2, batch=bt, stride_a=M * K, stride_b=N * K,
            stride_d=M * N, epi=nc.EPI_RESID_F32, aux=dev_f32(R), stride_aux=M * N)
    t.cuda.synchronize()
    for i in range(bt):
        acc = oracle.matmul_nt(A[i], B[i])
        assert rel_fro(host(D[i]), -0.5 * acc + 1.5 * Aux[i]) < 5e-3
        assert rel_fro(host(D2[i]), R[i] + acc) < 2e-5


@pytest.mark.parametrize("split", [1, 3, 7])
def test_gemm_split_k_accumulates(split):
    t = torch()
    M, N, K = 256, 256, 2048
    A = inputs.bf16_normal(9, (K, M))   # stored M-major, like dy^T
    B = inputs.bf16_normal(10, (K, N))  # stored N-major, like x
    D0 = np.random.default_rng(11).standard_normal((M, N)).astype(np.float32)
    D = dev_f32(D0)
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D, a_kmajor=0, b_kmajor=0, epi=nc.EPI_ACC_F32,
            split_k=split)
    t.cuda.synchronize()
    assert rel_fro(host(D), D0 + oracle.matmul_nt(A.T, B.T)) < 2e-5


def test_gemm_batched_strided():
    t = torch()
    bt, M, N, K = 3, 136, 264, 192
    A = inputs.bf16_normal(12, (bt, M, K))
    B = inputs.bf16_normal(13, (bt, K, N))  # N-major per batch
    D = t.empty(bt, M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D, b_kmajor=0, batch=bt, stride_a=M * K,
            stride_b=K * N, stride_d=M * N)
    t.cuda.synchronize()
    for i in range(bt):
        assert rel_fro(host(D[i]), oracle.matmul_nt(A[i], B[i].T)) < 5e-3


def test_gemm_rejects_bad_arguments():
    t = torch()
    A = t.zeros(64, 60, dtype=t.bfloat16, device="cuda")
    D = t.zeros(64, 64, dtype=t.bfloat16, device="cuda")
    with pytest.raises(nc.NcError) as e:
        nc.gemm(64, 64, 60, A, A, D, lda=60, ldb=60)  # 60 % 8 != 0
    assert e.value.status == nc.NC_ERR_INVALID_ARG
    with pytest.raises(nc.NcError):
        nc.gemm(64, 64, 64, A, A, D, epi=nc.EPI_STORE_BF16, split_k=2)


def test_gemm_full_size_sampled():
    """The MLP-up shape of the depth-20 step (65536 x 5120 x 1280, the size
    the step runs), checked on sampled rows and columns."""
    t = torch()
    M, N, K = 65536, 5120, 1280
    A = inputs.bf16_normal(14, (M, K))
    B = inputs.bf16_normal(15, (N, K), std=K ** -0.5)
    D = t.empty(M, N, dtype=t.bfloat16, device="cuda")
    nc.gemm(M, N, K, dev_bf16(A), dev_bf16(B), D, epi=nc.EPI_RELU2)
    t.cuda.synchronize()
    rng = np.random.default_rng(16)
    rows = np.sort(rng.choice(M, 96, replace=False))
    rows[-1] = M - 1
    cols = np.sort(rng.choice(N, 96, replace=False))
    ref = np.maximum(oracle.matmul_nt(A[rows], B[cols]), 0) ** 2
    got = host(D[t.from_numpy(rows).cuda()][:, t.from_numpy(cols).cuda()])
    assert rel_fro(got, ref) < 5e-3


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("rows,cols", [(1, 256), (37, 1280), (1000, 768)])
def test_rmsnorm(rows, cols):
    t = torch()
    x = (np.random.default_rng(17).standard_normal((rows, cols)) * 3).astype(np.float32)
    y = t.empty(rows, cols, dtype=t.bfloat16, device="cuda")
    r = t.empty(rows, dtype=t.float32, device="cuda")
    nc.rmsnorm(dev_f32(x), y, r, rows, cols)
    t.cuda.synchronize()
    yr, rr = oracle.rmsnorm(x)
    assert rel_fro(host(y), yr) < 5e-3
    np.testing.assert_allclose(host(r), rr, rtol=1e-5)


# ------------------------------------------------------------------ embedding gather
@pytest.mark.parametrize("ids", ["uniform", "zipf"])
def test_embed_gather_is_bit_exact(ids):
    """x = E[tok] bit for bit at the step's size (65536 ids, d = 1280, V =
    32768) through the gather kernel the model's forward launches; E holds
    full fp32 mantissas, so any conversion or partial copy would show."""
    t = torch()
    N, d, V = 65536, 1280, 32768
    if ids == "uniform":
        tok, _ = inputs.token_batch(80, 32, 2048)
    else:
        tok, _ = inputs.zipf_token_batch(81, 32, 2048)
    tok = tok.reshape(-1)
    assert tok.min() >= 0 and tok.max() < V
    E = np.random.default_rng(82).standard_normal((V, d)).astype(np.float32)
    Ed = t.from_numpy(E).cuda()
    x = t.full((N, d), float("nan"), dtype=t.float32, device="cuda")
    nc.embed_gather(t.from_numpy(tok).cuda(), N, Ed, V, d, x)
    nc.op_sync()
    assert np.array_equal(x.cpu().numpy().view(np.uint32), E[tok].view(np.uint32))


def test_embed_gather_out_of_range_ids_are_clamped_and_reported():
    """Ids below 0 read row 0 and ids at or above V read row V - 1 (nothing
    out of bounds); the op status word turns them into NC_ERR_TOKEN_RANGE at
    the next op_sync, which also clears it."""
    t = torch()
    V, d = 1000, 256
    tok = np.array([3, -1, 999, 1000, 5, -7, 123456, 0], dtype=np.int32)
    E = np.random.default_rng(83).standard_normal((V, d)).astype(np.float32)
    x = t.empty((len(tok), d), dtype=t.float32, device="cuda")
    nc.op_sync()  # nothing pending
    nc.embed_gather(t.from_numpy(tok).cuda(), len(tok), t.from_numpy(E).cuda(), V, d, x)
    with pytest.raises(nc.NcError) as e:
        nc.op_sync()
    assert e.value.status == nc.NC_ERR_TOKEN_RANGE
    nc.op_sync()  # cleared
    expect = E[np.clip(tok, 0, V - 1)]
    assert np.array_equal(x.cpu().numpy(), expect)


def test_exp2_poly_relative_error():
    """The softmax's FMA-pipe exponential on the GPU against exact 2^x (fp64):
    relative error within the polynomial's 7.5e-5 plus fp32 rounding over
    the softmax's range, integers exact up to the polynomial's value at 0,
    and arguments below -125 (masked scores: -inf) held near 2^-125."""
    t = torch()
    rng = np.random.default_rng(11)
    x = np.concatenate([np.linspace(-125.0, 20.0, 1 << 20), rng.uniform(-30.0, 1.0, 99_999),
                        np.arange(-125, 21, dtype=np.float64)]).astype(np.float32)
    dx = dev_f32(x)
    y = t.empty_like(dx)
    nc.exp2_poly(dx, y, x.size)  # odd length: the last thread takes one element
    t.cuda.synchronize()
    got = host(y).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 7.5e-5 + 2e-7
    special = np.array([-np.inf, -1e30, -126.0, -200.0], dtype=np.float32)
    ds = dev_f32(special)
    ys = t.empty_like(ds)
    nc.exp2_poly(ds, ys, special.size)
    t.cuda.synchronize()
    v = host(ys)
    assert np.all(np.isfinite(v)) and np.all(v > 0) and np.all(v < 2.0 ** -124)
    with pytest.raises(nc.NcError):
        nc.exp2_poly(ds, ys, -1)


# ------------------------------------------------------------------ fp8 (E4M3)
def _e4m3_decode(q):
    """Values of E4M3 bytes from the format's definition: sign bit, 4-bit
    exponent with bias 7, 3-bit mantissa; exponent 0 is subnormal (m * 2^-9);
    0x7f / 0xff are NaN."""
    b = np.arange(256)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e, m = (b >> 3) & 0xF, b & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7.0)) * sign
    val[(b & 0x7F) == 0x7F] = np.nan
    return val[np.asarray(q, dtype=np.int64)]


def _fp8_oracle_q(x, activation):
    """The oracle's quantised values of x: scale s = oracle.fp8_scale, then
    E4M3 of the fp32 product x * s (oracle.e4m3_round)."""
    s = np.float32(oracle.fp8_scale(x, activation=activation))
    return s, oracle.e4m3_round((np.float32(x) * s).astype(np.float64))


@pytest.mark.parametrize("bf16,transpose", [(True, False), (True, True), (False, False), (False, True)])
def test_fp8_quantize_is_bit_exact(bf16, transpose):
    t = torch()
    rows, cols = 80, 208  # ragged against the 64 x 64 transpose tiles
    x = inputs.bf16_normal(5, (rows, cols)) * 3.0
    x[3, 7] = 0.0
    x[10, :8] = [1e-4, -2e-3, 5e-3, 0.3, -7.0, 12.5, -0.0, 0.011]  # subnormal and normal codes
    x = inputs.round_to_bf16(x.astype(np.float32))  # the same numbers on both paths
    dx = dev_bf16(x) if bf16 else dev_f32(x)
    q = t.zeros((cols, rows) if transpose else (rows, cols), dtype=t.uint8, device="cuda")
    sc = t.zeros(2, dtype=t.float32, device="cuda")
    scratch = t.zeros(1, dtype=t.int32, device="cuda")
    nc.fp8_quantize(dx, rows, cols, q, sc, scratch, transpose=transpose)
    t.cuda.synchronize()
    s_ref, q_ref = _fp8_oracle_q(x, activation=bf16)
    assert np.float32(host(sc)[0]) == s_ref
    got = _e4m3_decode(host(q))
    assert np.array_equal(got.T if transpose else got, q_ref)
    # Saturation: the largest magnitude lands on 448 exactly.
    assert np.nanmax(np.abs(got)) == 448.0


def test_fp8_quantize_both_layouts_in_one_pass():
    """The one-pass form (both layouts, 64 x 128 tiles, ragged here) gives
    the single-layout op's bytes and scale, which match the oracle."""
    t = torch()
    rows, cols = 200, 328
    x = inputs.round_to_bf16((inputs.bf16_normal(7, (rows, cols)) * 5.0).astype(np.float32))
    dx = dev_bf16(x)
    q = t.zeros((rows, cols), dtype=t.uint8, device="cuda")
    qT = t.zeros((cols, rows), dtype=t.uint8, device="cuda")
    q1 = t.zeros((rows, cols + 8), dtype=t.uint8, device="cuda")
    sc = t.zeros(2, dtype=t.float32, device="cuda")
    scratch = t.zeros(2, dtype=t.int32, device="cuda")
    nc.fp8_quantize2(dx, rows, cols, q, qT, sc[0:1], scratch[0:1])
    nc.fp8_quantize(dx, rows, cols, q1, sc[1:2], scratch[1:2], ldq=cols + 8)
    t.cuda.synchronize()
    s = host(sc)
    assert s[0] == s[1] == np.float32(oracle.fp8_scale(x, activation=True))
    assert np.array_equal(host(q), host(q1)[:, :cols])
    assert np.array_equal(host(qT), host(q).T)
    _, q_ref = _fp8_oracle_q(x, activation=True)
    assert np.array_equal(_e4m3_decode(host(q)), q_ref)


@pytest.mark.parametrize("M,N,K,epi", [(512, 768, 640, "f32"), (300, 512, 1000, "f32"),
                                       (640, 1280, 1280, "bf16"), (384, 256, 256, "resid")])
def test_fp8_gemm_matches_the_oracle(M, N, K, epi):
    """y = x W^T on E4M3 operands (x an activation, W a weight), each with its
    own scale, against the oracle's fp64 product of the same quantised
    values; ragged M and K included.  The tensor cores sum the exact E4M3
    products in fp32, so the fp32 output is within 1e-5 (relative Frobenius)
    and the bf16 output within one bf16 rounding."""
    t = torch()
    x = inputs.bf16_normal(11, (M, K))
    w = (inputs.bf16_normal(12, (N, K)) * K ** -0.5).astype(np.float32)
    Kp = (K + 15) // 16 * 16
    qx = t.zeros((M, Kp), dtype=t.uint8, device="cuda")
    qw = t.zeros((N, Kp), dtype=t.uint8, device="cuda")
    sc = t.zeros(2, dtype=t.float32, device="cuda")
    scratch = t.zeros(2, dtype=t.int32, device="cuda")
    nc.fp8_quantize(dev_bf16(x), M, K, qx, sc[0:1], scratch[0:1], ldq=Kp)
    nc.fp8_quantize(dev_f32(w), N, K, qw, sc[1:2], scratch[1:2], ldq=Kp)
    ref = oracle.fp8_matmul_nt(x, w)
    if epi == "resid":
        R = inputs.bf16_normal(13, (M, N)).astype(np.float32)
        D = dev_f32(R)
        nc.gemm(M, N, K, qx, qw, D, lda=Kp, ldb=Kp, epi=nc.EPI_RESID_F32, aux=D, ab_scale=sc)
        ref = ref + R
    else:
        D = t.zeros(M, N, dtype=t.float32 if epi == "f32" else t.bfloat16, device="cuda")
        nc.gemm(M, N, K, qx, qw, D, lda=Kp, ldb=Kp,
                epi=nc.EPI_STORE_F32 if epi == "f32" else nc.EPI_STORE_BF16, ab_scale=sc)
    t.cuda.synchronize()
    assert rel_fro(host(D), ref) < (5e-3 if epi == "bf16" else 1e-5)


def test_fp8_gemm_weight_gradient_form():
    """dW = dy^T x (split K, fp32 accumulate) from transposed E4M3 copies of
    both activations (K = tokens), against the oracle's quantised product."""
    t = torch()
    rows, n, k = 1024, 384, 256
    dy = inputs.bf16_normal(21, (rows, n))
    x = inputs.bf16_normal(22, (rows, k))
    qd = t.zeros((n, rows), dtype=t.uint8, device="cuda")
    qx = t.zeros((k, rows), dtype=t.uint8, device="cuda")
    sc = t.zeros(2, dtype=t.float32, device="cuda")
    scratch = t.zeros(2, dtype=t.int32, device="cuda")
    nc.fp8_quantize(dev_bf16(dy), rows, n, qd, sc[0:1], scratch[0:1], transpose=True)
    nc.fp8_quantize(dev_bf16(x), rows, k, qx, sc[1:2], scratch[1:2], transpose=True)
    D = t.zeros(n, k, dtype=t.float32, device="cuda")
    nc.gemm(n, k, rows, qd, qx, D, epi=nc.EPI_ACC_F32, split_k=0, ab_scale=sc)
    t.cuda.synchronize()
    ref = oracle.fp8_matmul_nt(np.ascontiguousarray(dy.T), np.ascontiguousarray(x.T))
    assert rel_fro(host(D), ref) < 1e-5


@pytest.mark.parametrize("epi", ["relu2", "relu2_bwd"])
def test_fp8_gemm_amax_out_is_the_outputs_max(epi):
    """amax_out receives max |D| over the bf16 values the epilogue stored."""
    t = torch()
    M, N, K = 384, 512, 256
    x = inputs.bf16_normal(31, (M, K))
    w = inputs.bf16_normal(32, (N, K)) * K ** -0.5
    qx = t.zeros((M, K), dtype=t.uint8, device="cuda")
    qw = t.zeros((N, K), dtype=t.uint8, device="cuda")
    sc = t.zeros(2, dtype=t.float32, device="cuda")
    scratch = t.zeros(2, dtype=t.int32, device="cuda")
    nc.fp8_quantize(dev_bf16(x), M, K, qx, sc[0:1], scratch[0:1])
    nc.fp8_quantize(dev_f32(w), N, K, qw, sc[1:2], scratch[1:2])
    D = t.zeros(M, N, dtype=t.bfloat16, device="cuda")
    amax = t.zeros(1, dtype=t.int32, device="cuda")
    aux = dev_bf16(np.abs(inputs.bf16_normal(33, (M, N)))) if epi == "relu2_bwd" else None
    nc.gemm(M, N, K, qx, qw, D, epi=nc.EPI_RELU2 if epi == "relu2" else nc.EPI_RELU2_BWD, aux=aux,
            ab_scale=sc, amax_out=amax)
    t.cuda.synchronize()
    got = amax.cpu().numpy().view(np.float32)[0]
    assert got == np.abs(host(D)).max() > 0


def test_fp8_gemm_rejects_unsupported_forms():
    t = torch()
    q = t.zeros((512, 512), dtype=t.uint8, device="cuda")
    sc = t.ones(2, dtype=t.float32, device="cuda")
    D = t.zeros(512, 512, dtype=t.float32, device="cuda")
    with pytest.raises(nc.NcError):
        nc.gemm(512, 512, 512, q, q, D, a_kmajor=False, epi=nc.EPI_STORE_F32, ab_scale=sc)
    with pytest.raises(nc.NcError):
        nc.gemm(512, 512, 512, q, q, D, epi=nc.EPI_STORE_F32, alpha=2.0, ab_scale=sc)
    with pytest.raises(nc.NcError):
        nc.gemm(100, 512, 512, q, q, D, epi=nc.EPI_STORE_F32, ab_scale=sc)  # M <= 128


def test_planted_op_status_is_reported_once():
    """An expired bounded wait inside an op (planted here as its status code,
    not produced by a stuck kernel) surfaces as NC_ERR_TIMEOUT at the next
    op_sync and is cleared by it."""
    t = torch()
    ptr = nc.lib().nc_debug_op_status_word()
    assert ptr

    class _Word:
        __cuda_array_interface__ = {"shape": (1,), "typestr": "<i4", "data": (ptr, False),
                                    "version": 3}

    word = t.as_tensor(_Word(), device="cuda")
    nc.op_sync()
    word.fill_(1)
    t.cuda.synchronize()
    with pytest.raises(nc.NcError) as e:
        nc.op_sync()
    assert e.value.status == nc.NC_ERR_TIMEOUT
    nc.op_sync()


# ------------------------------------------------------------------ attention
def _attn_inputs(B, T, H, seed):
    # q, k with unit RMS per head (as after QK-norm), v normal; fused [B*T, 3d] rows.
    d = H * 128
    qkv = inputs.bf16_normal(seed, (B * T, 3 * d))
    return qkv


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 200, 2), (1, 1, 1), (1, 577, 3)])
def test_attention_forward(B, T, H):
    t = torch()
    d = H * 128
    qkv = _attn_inputs(B, T, H, 18 + T)
    q = qkv[:, :d].reshape(B, T, H, 128)
    k = qkv[:, d:2 * d].reshape(B, T, H, 128)
    v = qkv[:, 2 * d:].reshape(B, T, H, 128)
    dq = dev_bf16(qkv)
    o = t.empty(B * T, d, dtype=t.bfloat16, device="cuda")
    lse = t.empty(B, H, T, dtype=t.float32, device="cuda")
    nc.attention_fwd(dq, dq[:, d:], dq[:, 2 * d:], 3 * d, o, d, lse, B, T, H)
    t.cuda.synchronize()
    oref, lref, _ = oracle.attention(q, k, v)
    assert rel_fro(host(o), oref.reshape(B * T, d)) < 5e-3
    np.testing.assert_allclose(host(lse), lref, rtol=2e-4, atol=2e-4)


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 200, 2), (1, 333, 1)])
def test_attention_backward(B, T, H):
    t = torch()
    d = H * 128
    qkv = _attn_inputs(B, T, H, 40 + T)
    q = qkv[:, :d].reshape(B, T, H, 128)
    k = qkv[:, d:2 * d].reshape(B, T, H, 128)
    v = qkv[:, 2 * d:].reshape(B, T, H, 128)
    # The backward consumes the forward's O and lse; those come from the
    # oracle here (rounded to bf16 like the saved activation).
    oref, lref, _ = oracle.attention(q, k, v)
    o_b = inputs.round_to_bf16(oref.reshape(B * T, d).astype(np.float32))
    dout = inputs.bf16_normal(41 + T, (B * T, d))
    dqkv = t.zeros(B * T, 3 * d, dtype=t.bfloat16, device="cuda")
    dqf = t.empty(B * T, d, dtype=t.float32, device="cuda")
    delta = t.empty(B, H, T, dtype=t.float32, device="cuda")
    tq = dev_bf16(qkv)
    nc.attention_bwd(tq, tq[:, d:], tq[:, 2 * d:], 3 * d, dev_bf16(o_b), dev_bf16(dout), d,
                     dev_f32(lref.astype(np.float32)), dqf, dqkv[:, d:], dqkv[:, 2 * d:], 3 * d,
                     delta, B, T, H)
    t.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd(q, k, v, lref, dout.reshape(B, T, H, 128))
    assert rel_fro(host(dqf), rq.reshape(B * T, d)) < 1e-2
    assert rel_fro(host(dqkv[:, d:2 * d]), rk.reshape(B * T, d)) < 1e-2
    assert rel_fro(host(dqkv[:, 2 * d:]), rv.reshape(B * T, d)) < 1e-2


@pytest.mark.parametrize("B,T,H,Hkv,window", [(1, 300, 4, 2, 100),   # window inside one tile
                                               (2, 333, 2, 1, 129),   # just past a tile
                                               (1, 520, 4, 1, 0),     # self only, one KV head
                                               (1, 256, 3, 3, -1),    # no window, no groups
                                               (1, 700, 2, 2, 255)])
def test_attention_grouped_kv_and_window(B, T, H, Hkv, window):
    """Causal attention with Hkv KV heads and a left window, forward and
    backward, against the oracle's grouped / windowed attention."""
    t = torch()
    dq_, dkv_ = H * 128, Hkv * 128
    width = dq_ + 2 * dkv_
    qkv = inputs.bf16_normal(70 + T + window, (B * T, width))
    q = qkv[:, :dq_].reshape(B, T, H, 128)
    k = qkv[:, dq_:dq_ + dkv_].reshape(B, T, Hkv, 128)
    v = qkv[:, dq_ + dkv_:].reshape(B, T, Hkv, 128)
    dev = dev_bf16(qkv)
    o = t.empty(B * T, dq_, dtype=t.bfloat16, device="cuda")
    lse = t.empty(B, H, T, dtype=t.float32, device="cuda")
    nc.attention_fwd_ex(dev, width, dev[:, dq_:], dev[:, dq_ + dkv_:], width, o, dq_, lse, B, T, H,
                        Hkv, window)
    t.cuda.synchronize()
    oref, lref = oracle.attention_ex(q, k, v, window=window)
    assert rel_fro(host(o), oref.reshape(B * T, dq_)) < 5e-3
    np.testing.assert_allclose(host(lse), lref, rtol=2e-4, atol=2e-4)
    # Backward from the oracle's O and lse (O rounded to bf16 like the saved activation).
    o_b = inputs.round_to_bf16(oref.reshape(B * T, dq_).astype(np.float32))
    dout = inputs.bf16_normal(71 + T, (B * T, dq_))
    dqf = t.empty(B * T, dq_, dtype=t.float32, device="cuda")
    dkv = t.zeros(B * T, 2 * dkv_, dtype=t.bfloat16, device="cuda")
    delta = t.empty(B, H, T, dtype=t.float32, device="cuda")
    nc.attention_bwd_ex(dev, width, dev[:, dq_:], dev[:, dq_ + dkv_:], width, dev_bf16(o_b),
                        dev_bf16(dout), dq_, dev_f32(lref.astype(np.float32)), dqf, dkv[:, :dkv_],
                        dkv[:, dkv_:], 2 * dkv_, delta, B, T, H, Hkv, window)
    t.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd_ex(q, k, v, lref, dout.reshape(B, T, H, 128), window=window)
    assert rel_fro(host(dqf), rq.reshape(B * T, dq_)) < 1e-2
    assert rel_fro(host(dkv[:, :dkv_]), rk.reshape(B * T, dkv_)) < 1e-2
    assert rel_fro(host(dkv[:, dkv_:]), rv.reshape(B * T, dkv_)) < 1e-2


def test_attention_full_length_sampled_heads():
    """T = 2048 (the step's sequence length), one batch row, two heads."""
    t = torch()
    B, T, H = 1, 2048, 2
    d = H * 128
    qkv = _attn_inputs(B, T, H, 60)
    dq = dev_bf16(qkv)
    o = t.empty(B * T, d, dtype=t.bfloat16, device="cuda")
    lse = t.empty(B, H, T, dtype=t.float32, device="cuda")
    nc.attention_fwd(dq, dq[:, d:], dq[:, 2 * d:], 3 * d, o, d, lse, B, T, H)
    t.cuda.synchronize()
    q = qkv[:, :d].reshape(B, T, H, 128)
    k = qkv[:, d:2 * d].reshape(B, T, H, 128)
    v = qkv[:, 2 * d:].reshape(B, T, H, 128)
    oref, lref, _ = oracle.attention(q, k, v)
    assert rel_fro(host(o), oref.reshape(B * T, d)) < 5e-3
    np.testing.assert_allclose(host(lse), lref, rtol=2e-4, atol=2e-4)


def test_attention_backward_full_length():
    """The backward at the step's sequence length, T = 2048 (16 key tiles,
    each looping over up to 16 query tiles), one batch row, two heads,
    against the oracle's backward from the oracle's O and lse."""
    t = torch()
    B, T, H = 1, 2048, 2
    d = H * 128
    qkv = _attn_inputs(B, T, H, 61)
    q = qkv[:, :d].reshape(B, T, H, 128)
    k = qkv[:, d:2 * d].reshape(B, T, H, 128)
    v = qkv[:, 2 * d:].reshape(B, T, H, 128)
    oref, lref, _ = oracle.attention(q, k, v)
    o_b = inputs.round_to_bf16(oref.reshape(B * T, d).astype(np.float32))
    dout = inputs.bf16_normal(62, (B * T, d))
    dqkv = t.zeros(B * T, 3 * d, dtype=t.bfloat16, device="cuda")
    dqf = t.empty(B * T, d, dtype=t.float32, device="cuda")
    delta = t.empty(B, H, T, dtype=t.float32, device="cuda")
    tq = dev_bf16(qkv)
    nc.attention_bwd(tq, tq[:, d:], tq[:, 2 * d:], 3 * d, dev_bf16(o_b), dev_bf16(dout), d,
                     dev_f32(lref.astype(np.float32)), dqf, dqkv[:, d:], dqkv[:, 2 * d:], 3 * d,
                     delta, B, T, H)
    t.cuda.synchronize()
    rq, rk, rv = oracle.attention_bwd(q, k, v, lref, dout.reshape(B, T, H, 128))
    assert rel_fro(host(dqf), rq.reshape(B * T, d)) < 1e-2
    assert rel_fro(host(dqkv[:, d:2 * d]), rk.reshape(B * T, d)) < 1e-2
    assert rel_fro(host(dqkv[:, 2 * d:]), rv.reshape(B * T, d)) < 1e-2


# ------------------------------------------------------------------ Newton-Schulz
@pytest.mark.parametrize("count,rows,cols", [(3, 256, 256), (2, 128, 512), (2, 512, 128),
                                             (2, 640, 640), (1, 768, 1536)])
def test_newton_schulz_op(count, rows, cols):
    """Five Newton-Schulz steps against the oracle.  From 2 x 2 tiles of 256
    up, the two symmetric products (X X^T and b A + c A A) compute only the
    tiles on or above the diagonal and store the others transposed; 640
    leaves ragged edge tiles on both sides."""
    t = torch()
    X = inputs.normal_stack(70 + rows, count, rows, cols)
    out = t.empty(count, rows, cols, dtype=t.bfloat16, device="cuda")
    scratch = t.empty(nc.newton_schulz_scratch_bytes(count, rows, cols), dtype=t.uint8,
                      device="cuda")
    nc.newton_schulz(dev_bf16(X), out, count, rows, cols, 5, scratch)
    t.cuda.synchronize()
    got = host(out)
    for i in range(count):
        ref = oracle.newton_schulz(X[i])
        assert rel_fro(got[i], ref) < 2e-2
        s = np.linalg.svd(got[i], compute_uv=False)
        if rows != cols:  # wide/tall N(0,1): every normalised sigma is well above 2e-3
            assert s.min() > 0.6 and s.max() < 1.22


@pytest.mark.parametrize("M,H,T", [(300, 2, 100), (256, 1, 256), (130, 3, 64)])
def test_gemm_rope_qknorm_epilogue(M, H, T):
    """q|k|v projection with RoPE + QK-norm fused into the GEMM epilogue,
    against the oracle's matmul, rotation and RMSNorm applied per head."""
    t = torch()
    d = 128 * H
    K = d
    X = inputs.bf16_normal(80 + M, (M, K))
    W = inputs.bf16_normal(81 + M, (3 * d, K), std=K ** -0.5)
    pos = np.arange(M) % T
    th = pos[:, None] * 10000.0 ** (-np.arange(64)[None, :] / 64.0)
    tab = np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32)  # [M, 64, 2]
    tab_dev = dev_f32(np.ascontiguousarray(tab[:T]))
    D = t.empty(M, 3 * d, dtype=t.bfloat16, device="cuda")
    rq = t.empty(M, H, dtype=t.float32, device="cuda")
    rk = t.empty(M, H, dtype=t.float32, device="cuda")
    desc = nc.GemmDesc()
    desc.M, desc.N, desc.K, desc.batch = M, 3 * d, K, 1
    tx, tw = dev_bf16(X), dev_bf16(W)
    desc.A, desc.lda, desc.a_kmajor = tx.data_ptr(), K, 1
    desc.B, desc.ldb, desc.b_kmajor = tw.data_ptr(), K, 1
    desc.D, desc.ldd = D.data_ptr(), 3 * d
    desc.epi, desc.alpha, desc.split_k = nc.EPI_ROPE_QKNORM, 1.0, 1
    desc.rope_T, desc.rope_H, desc.rope_tab = T, H, tab_dev.data_ptr()
    desc.rstd_q, desc.rstd_k = rq.data_ptr(), rk.data_ptr()
    nc._check(nc.lib().nc_op_gemm(desc, None))
    t.cuda.synchronize()
    ref = oracle.matmul_nt(X, W)
    expect = ref.copy()
    rstd = np.zeros((2, M, H))
    for which in range(2):
        for h in range(H):
            cols = slice(which * d + h * 128, which * d + (h + 1) * 128)
            rot = np.stack([oracle.rope_row(ref[m, cols], int(pos[m])) for m in range(M)])
            y, r = oracle.rmsnorm(rot)
            expect[:, cols] = y
            rstd[which, :, h] = r
    assert rel_fro(host(D), expect) < 5e-3
    np.testing.assert_allclose(host(rq), rstd[0], rtol=1e-4)
    np.testing.assert_allclose(host(rk), rstd[1], rtol=1e-4)
