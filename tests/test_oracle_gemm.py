"""Pins for oracle.gemm (CPU only).

gist.science technical summary, section 2.B: the compensated product recovers
FP32-level accuracy from 16-bit partial products; section 1: a plain 16-bit GEMM
whose FP32 result is stored as BF16 at the kernel boundary does not.
"""
from fractions import Fraction

import numpy as np
import pytest

import synthetic
from oracle import gemm as G
from oracle import split as S


def frac_matmul(A, B):
    A = [[Fraction(float(v)) for v in row] for row in np.asarray(A, np.float64)]
    B = [[Fraction(float(v)) for v in row] for row in np.asarray(B, np.float64)]
    n, k, m = len(A), len(B), len(B[0])
    return [[sum(A[i][t] * B[t][j] for t in range(k)) for j in range(m)] for i in range(n)]


def dyadic(shape, rng, bits=6):
    """Entries j / 2**bits with |j| < 2**9: exactly representable in FP16 and BF16."""
    return (rng.integers(-255, 256, size=shape) / float(1 << bits)).astype(np.float32)


@pytest.mark.parametrize("shape", [(2, 2, 2), (3, 5, 4), (8, 16, 8)])
@pytest.mark.parametrize("fmt", [S.FP16_S11, S.BF16])
def test_exact_on_16bit_representable_inputs(shape, fmt):
    n, k, m = shape
    rng = np.random.default_rng(n * 100 + k)
    A, B = dyadic((n, k), rng), dyadic((k, m), rng)
    exact = frac_matmul(A, B)
    ref = G.gemm_ref(A, B)
    emu = G.gemm_emulated(A, B, fmt)
    for i in range(n):
        for j in range(m):
            assert Fraction(float(ref[i, j])) == exact[i][j]
            assert Fraction(float(emu[i, j])) == exact[i][j]


@pytest.mark.parametrize("shape", [(2, 2, 2), (3, 5, 4), (8, 16, 8)])
def test_dropped_lo_lo_term_exactly(shape):
    """x = h + l * 2**-11 with both parts exact FP16 and |l| small: the split returns
    (h, l) and C_ref - C_emul is exactly 2**-22 * Al @ Bl (the only dropped term)."""
    n, k, m = shape
    rng = np.random.default_rng(11 + n)

    def make(shp):
        h = 1.0 + rng.integers(0, 1024, size=shp) / 1024.0          # FP16 values in [1, 2)
        l = rng.integers(-31, 32, size=shp) / 64.0                  # |l| < 0.5: within half an FP16 step of h
        return (h + l * 2.0 ** -11).astype(np.float32), h, l

    A, Ah, Al = make((n, k))
    B, Bh, Bl = make((k, m))
    hi, lo, _, _ = S.split(A, S.FP16_S11)
    np.testing.assert_array_equal(hi, Ah)
    np.testing.assert_array_equal(lo, Al)
    exact_ref = frac_matmul(A, B)
    exact_ll = frac_matmul(Al, Bl)
    emu = G.gemm_emulated(A, B, S.FP16_S11)
    for i in range(n):
        for j in range(m):
            want = exact_ref[i][j] - Fraction(1, 1 << 22) * exact_ll[i][j]
            assert Fraction(float(emu[i, j])) == want


@pytest.mark.parametrize("fmt", [S.FP16_S11, S.BF16])
def test_truncation_identity(fmt):
    X, W = synthetic.gemm_prefill(M=64, K=512, N=96)
    X, W = X.numpy(), W.numpy()
    ref = G.gemm_ref(X, W)
    emu = G.gemm_emulated(X, W, fmt)
    tt = G.truncation_term(X, W, fmt)
    scale = np.linalg.norm(ref)
    assert np.linalg.norm((emu - ref) - tt) <= 1e-12 * scale
    assert np.linalg.norm(tt) > 0


def test_error_levels_compensated_vs_downcast():
    A, B = synthetic.gemm_square(256, seed=0)
    A, B = A.numpy(), B.numpy()
    ref = G.gemm_ref(A, B)
    e_fp16 = G.normwise_rel_err(G.gemm_emulated(A, B, S.FP16_S11), ref)
    e_bf16 = G.normwise_rel_err(G.gemm_emulated(A, B, S.BF16), ref)
    e_down = G.normwise_rel_err(G.gemm_bf16_downcast(A, B), ref)
    # FP32 level for the scaled FP16 split: each operand carries ~22 bits
    assert 1e-8 < e_fp16 < 2e-7
    # BF16 hi/lo carries ~16 bits per operand: better than BF16, short of 1e-6
    assert 1e-6 < e_bf16 < 2e-5
    # the boundary downcast to BF16 costs ~2**-9 relative
    assert 1e-3 < e_down < 1e-2
    # the FP32-accumulated, unrounded product of BF16 operands is not enough either
    e_bf16_in = G.normwise_rel_err(
        S.to_bf16_as_f32(A).astype(np.float64) @ S.to_bf16_as_f32(B).astype(np.float64), ref)
    assert e_bf16_in > 1e-3


def test_channel_rescale_is_exact_and_prevents_overflow():
    rng = np.random.default_rng(3)
    A = rng.standard_normal((32, 64)).astype(np.float32)
    B = (0.02 * rng.standard_normal((64, 48))).astype(np.float32)
    A[:, 5] *= 1e5                                  # beyond FP16 range
    ref = G.gemm_ref(A, B)
    with np.errstate(invalid="ignore", over="ignore"):
        bad = G.gemm_emulated(A, B, S.FP16_S11)
    assert not np.all(np.isfinite(bad))
    e = G.suggest_channel_exponents(A)
    assert e[5] > 0 and np.count_nonzero(e) == 1
    As, Bs = G.rescale_channels(A, B, e)
    np.testing.assert_array_equal(G.gemm_ref(As, Bs), ref)           # power-of-two rescale is exact
    good = G.gemm_emulated(A, B, S.FP16_S11, chan_exp=e)
    assert G.normwise_rel_err(good, ref) < 2e-7


def test_gemm_ref_matches_scalar_loop():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((4, 37)).astype(np.float32)
    B = rng.standard_normal((37, 3)).astype(np.float32)
    ref = G.gemm_ref(A, B)
    for i in range(4):
        for j in range(3):
            exact = sum(Fraction(float(A[i, t])) * Fraction(float(B[t, j])) for t in range(37))
            assert abs(float(exact) - ref[i, j]) <= 1e-13 * max(1.0, abs(float(exact)))


@pytest.mark.parametrize("shape", [(2, 3, 2), (4, 8, 3)])
@pytest.mark.parametrize("fmt", [S.FP16_S11, S.BF16])
def test_two_product_identity_exact(shape, fmt):
    """Two-product form (technical summary 2.B): only A is split and the 16-bit weights carry
    no residual.  Exact rational check of C_two - A @ W16 = -Ar @ W16 with Ar = A - Ah - s Al,
    on random FP32 A (whose split leaves a nonzero Ar) and dyadic 16-bit weights."""
    n, k, m = shape
    rng = np.random.default_rng(7 * n + k)
    A = rng.standard_normal((n, k)).astype(np.float32)
    W16 = dyadic((k, m), rng)
    two = G.gemm_two_product(A, W16, fmt)
    Ah, Al, _, _ = S.split(A, fmt)
    s = Fraction(1) / Fraction(int(S.LO_SCALE[fmt]))
    exactA = [[Fraction(float(v)) for v in row] for row in A.astype(np.float64)]
    emulA = [[Fraction(float(Ah[i, t])) + s * Fraction(float(Al[i, t])) for t in range(k)] for i in range(n)]
    Wf = [[Fraction(float(v)) for v in row] for row in W16.astype(np.float64)]
    assert any(exactA[i][t] != emulA[i][t] for i in range(n) for t in range(k)), "Ar must be nonzero somewhere"
    trunc = G.two_product_truncation(A, W16, fmt)
    for i in range(n):
        for j in range(m):
            c_emul = sum(emulA[i][t] * Wf[t][j] for t in range(k))
            c_exact = sum(exactA[i][t] * Wf[t][j] for t in range(k))
            # the float64 evaluation of the small dyadic products is exact
            assert Fraction(float(two[i, j])) == c_emul
            assert abs(float(trunc[i, j]) - float(c_emul - c_exact)) <= 1e-15 * max(1.0, abs(float(c_exact)))


def test_two_product_error_levels():
    """Against the product with the 16-bit weights, the two-product form is at the level of
    the activation split (FP16: ~1e-7; BF16: ~1e-5); against the FP32 weights it is limited
    by the 16-bit rounding of the weights themselves (~1e-4 for FP16)."""
    X, W = synthetic.gemm_decode(16, K=512, N=256)
    X, W = X.numpy(), W.numpy()
    W16 = G.to_16bit(W, S.FP16_S11)
    e16 = G.normwise_rel_err(G.gemm_two_product(X, W16, S.FP16_S11), G.gemm_ref(X, W16))
    assert e16 < 2e-7
    Wb = G.to_16bit(W, S.BF16)
    eb = G.normwise_rel_err(G.gemm_two_product(X, Wb, S.BF16), G.gemm_ref(X, Wb))
    assert 1e-7 < eb < 2e-5
    e_w = G.normwise_rel_err(G.gemm_two_product(X, W16, S.FP16_S11), G.gemm_ref(X, W))
    assert 1e-5 < e_w < 1e-3


def test_bf16_downcast_exact_dyadic_cases():
    """Hand-worked values of the boundary-truncation control (technical summary, section 1:
    FP32 accumulators written to BF16 memory).  BF16 keeps 7 stored mantissa bits: the
    spacing is 2^-7 in [1, 2) and 2^-6 in [2, 4)."""
    d = 2.0 ** -10
    # (a) the inputs are rounded first: 1 + 3*2^-10 lies below the half-way point 1 + 2^-8,
    #     so each rounds to 1 and C = 3; the unrounded sum 3 + 9*2^-10 would have rounded up
    #     to 3 + 2^-6 on the BF16 store
    A = np.array([[1 + 3 * d, 1 + 3 * d, 1 + 3 * d]], np.float32)
    B = np.ones((3, 1), np.float32)
    assert G.gemm_bf16_downcast(A, B)[0, 0] == 3.0
    # (b) the result is rounded on the store, ties to even: 1 + 1.5*2^-7 sits half-way
    #     between 1 + 2^-7 (odd last bit) and 1 + 2^-6 (even), so it stores as 1 + 2^-6
    A = np.ones((1, 3), np.float32)
    B = np.array([[1.0], [2.0 ** -7], [2.0 ** -8]], np.float32)
    assert G.gemm_bf16_downcast(A, B)[0, 0] == 1.0 + 2.0 ** -6
    #     and 1 + 2^-8, half-way between 1 (even) and 1 + 2^-7, stores as 1
    B = np.array([[1.0], [2.0 ** -9], [2.0 ** -9]], np.float32)
    assert G.gemm_bf16_downcast(A, B)[0, 0] == 1.0
    # (c) orientation: BF16-exact small integers with exact sums give C = A @ B, written out
    A = np.array([[1, 2, 0], [-3, 1, 4]], np.float32)
    B = np.array([[2, -1], [0, 5], [1, 3]], np.float32)
    np.testing.assert_array_equal(G.gemm_bf16_downcast(A, B), [[2.0, 9.0], [-2.0, 20.0]])
