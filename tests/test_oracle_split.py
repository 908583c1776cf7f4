"""Pins for oracle.split against the exact nearest-value definition (CPU only).

The split follows the gist.science technical summary, section 2.B (primary 16-bit
value plus residual), read as round-to-nearest-even FP16 hi and a 2**11-scaled FP16
lo (or BF16 hi / unscaled BF16 lo).
"""
import numpy as np
import pytest

from oracle import split as S


def nearest_even(v, mant_bits, emin, max_finite):
    """Independent round-to-nearest-even onto a binary format with ``mant_bits``
    stored mantissa bits and minimum normal exponent ``emin`` (integer arithmetic in
    float64, no dtype casts)."""
    v = np.asarray(v, np.float64)
    out = np.zeros_like(v)
    nz = v != 0
    _, e = np.frexp(np.abs(v[nz]))          # |v| = f * 2**e, f in [0.5, 1)
    e = np.maximum(e - 1, emin)             # exponent of the leading bit (clamped to subnormal range)
    spacing = np.ldexp(1.0, e - mant_bits)
    n = v[nz] / spacing                     # exact (power-of-two scaling)
    fl = np.floor(n)
    frac = n - fl
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(fl, 2) == 1))
    r = (fl + up) * spacing
    r = np.where(np.abs(r) > max_finite, np.copysign(np.inf, r), r)
    out[nz] = r
    return out


def fp16_nearest(v):
    return nearest_even(v, 10, -14, 65504.0)


def bf16_nearest(v):
    return nearest_even(v, 7, -126, float(np.finfo(np.float32).max))


def mantissa_sweep(exponent, sign=1.0, step=1):
    m = np.arange(0, 1 << 23, step, dtype=np.int64)
    bits = ((exponent + 127) << 23) | m
    x = bits.astype(np.uint32).view(np.float32)
    return (sign * x).astype(np.float32)


@pytest.mark.parametrize("exponent", [0, -5, 10, -17])
@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_fp16_s11_hi_lo_are_nearest_even(exponent, sign):
    x = mantissa_sweep(exponent, sign, step=1 if exponent == 0 else 5)
    hi, lo, _, _ = S.split(x, S.FP16_S11)
    np.testing.assert_array_equal(hi, fp16_nearest(x))
    r = x.astype(np.float64) - hi
    np.testing.assert_array_equal(lo, fp16_nearest(r * 2048.0))


@pytest.mark.parametrize("exponent", [0, -5, 10, -17])
def test_fp16_s11_reconstruction_bound(exponent):
    x = mantissa_sweep(exponent, 1.0, step=3)
    hi, lo, _, _ = S.split(x, S.FP16_S11)
    err = np.abs(x.astype(np.float64) - S.reconstruct(hi, lo, S.FP16_S11))
    bound = np.maximum(2.0 ** -22 * np.abs(x.astype(np.float64)), 2.0 ** -36)
    assert np.all(err <= bound)
    # the remainder is genuinely below hi's own rounding error (the residual term adds bits)
    assert np.all(err <= np.abs(x.astype(np.float64) - hi) + 0.0)


@pytest.mark.parametrize("exponent", [0, -5, 10, -60, 60])
def test_bf16_hi_lo_are_nearest_even(exponent):
    x = mantissa_sweep(exponent, -1.0 if exponent % 2 else 1.0, step=1 if exponent == 0 else 5)
    hi, lo, hb, lb = S.split(x, S.BF16)
    np.testing.assert_array_equal(hi, bf16_nearest(x))
    np.testing.assert_array_equal(lo, bf16_nearest(x.astype(np.float64) - hi))
    err = np.abs(x.astype(np.float64) - (hi + lo))
    assert np.all(err <= 2.0 ** -17 * np.abs(x.astype(np.float64)))
    # the encodings are the top 16 bits of the FP32 pattern of the same values
    np.testing.assert_array_equal(hb, (hi.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))


def test_fp16_special_values():
    x = np.array([0.0, -0.0, 65504.0, 65519.99, 2.0 ** -24, 2.0 ** -25, 1.0 + 2.0 ** -11,
                  1.0 + 3 * 2.0 ** -11, 65520.0, -70000.0], np.float32)
    hi, lo, _, _ = S.split(x, S.FP16_S11)
    assert hi[0] == 0 and lo[0] == 0
    assert hi[2] == 65504.0 and lo[2] == 0.0
    assert hi[3] == 65504.0 and lo[3] == pytest.approx((65519.99 - 65504.0) * 2048, rel=2 ** -10)
    assert hi[4] == 2.0 ** -24 and lo[4] == 0.0
    assert hi[5] == 0.0 and lo[5] == 2.0 ** -14          # tie at half the smallest subnormal -> even (0)
    assert hi[6] == 1.0 and lo[6] == 1.0                  # tie -> even hi, residual 2**-11 -> lo 1.0
    assert hi[7] == 1.0 + 2.0 ** -9 and lo[7] == -1.0     # tie -> even (rounds up), residual -2**-11
    assert np.isinf(hi[8]) and np.isinf(hi[9])            # beyond FP16 range: needs the channel rescale


def test_split_is_elementwise_and_deterministic():
    rng = np.random.default_rng(7)
    x = rng.standard_normal(1000).astype(np.float32)
    a = S.split(x, S.FP16_S11)
    b = S.split(x[::-1].copy(), S.FP16_S11)
    np.testing.assert_array_equal(a[2], b[2][::-1])
    np.testing.assert_array_equal(a[3], b[3][::-1])


def test_format_helpers_on_hand_worked_values():
    """FP16 / BF16 roundings and encodings that the split builds on, written out by hand."""
    # FP16 spacing in [1, 2) is 2^-10; half-way points go to the even neighbour
    x = np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 65504.0, 65520.0, 2.0 ** -24, 2.0 ** -25], np.float64)
    h = S.to_fp16(x)
    assert h.dtype == np.float16
    np.testing.assert_array_equal(h.astype(np.float64), [1.0, 1 + 2.0 ** -9, 65504.0, np.inf, 2.0 ** -24, 0.0])
    np.testing.assert_array_equal(h.view(np.uint16), [0x3C00, 0x3C02, 0x7BFF, 0x7C00, 0x0001, 0x0000])
    # BF16: 1 + 2^-8 is half-way between 1 and 1 + 2^-7 (odd) -> 1; 1 + 3*2^-8 -> 1 + 2^-6
    b = S.to_bf16_as_f32(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -2.5], np.float32))
    np.testing.assert_array_equal(b, [1.0, 1 + 2.0 ** -6, -2.5])
    np.testing.assert_array_equal(S.bf16_bits(b), [0x3F80, 0x3F82, 0xC020])
