"""Reference and emulated compensated GEMM (oracle; test infrastructure only).

Sources:
  * gist.science technical summary, section 2.B "Mitigating GEMM Truncation via
    Algebraic Error Compensation": operands split into a 16-bit primary value and a
    residual, partial products on 16-bit tensor cores with FP32 accumulation, summed.
    Same section, "Overflow Handling": targeted rescaling of rare outlier channels.
  * section 1 "Root Cause Analysis": the loss comes from writing FP32 accumulators
    to BF16 memory at kernel boundaries (the negative control below).
  * authors' v2 abstract: high-precision matrix multiplication synthesised on
    16-bit tensor cores by algebraic error compensation.

Functions:
  gemm_ref          C_ref = A @ B in float64 -- the exact product the method
                    approximates (definition; FP64 rounding only).
  gemm_emulated     C_emul = Ah Bh + s (Ah Bl + Al Bh), s = 1/lo_scale, evaluated
                    in float64 from the oracle's own split -- the method's steps.
                    (three products; the lo*lo term is dropped.)
  truncation_term   closed form of C_emul - C_ref from the split residuals.
  to_16bit          the 16-bit form of a weight matrix (FP16 or BF16 per the format).
  gemm_two_product  C = Ah W16 + s Al W16: the section's own two-product form, in which
                    only the activations are split and the weights are 16-bit values.
  two_product_truncation  closed form of gemm_two_product - A @ W16.
  gemm_bf16_downcast  plain 16-bit GEMM with a BF16 store of the FP32 result: the
                    boundary-truncation negative control.
  rescale_channels  per-K-channel power-of-two rescale (exact).
  normwise_rel_err  ||C - C_ref||_F / ||C_ref||_F.

Parity: pinned (exact rational brute force on dyadic inputs; the identity
C_emul - C_ref = truncation_term; error levels of the compensated product versus
the BF16 downcast control; exactness of the channel rescale).
"""
import numpy as np

from . import split as _split


def gemm_ref(A, B):
    """Exact-product reference: float64 matmul of the FP32 inputs."""
    return np.asarray(A, np.float64) @ np.asarray(B, np.float64)


def rescale_channels(A, B, chan_exp):
    """A[:, k] * 2**-e_k and B[k, :] * 2**e_k (power-of-two, so A @ B is unchanged).

    ``chan_exp`` is an int array of length K or None.  Returns float32 arrays.
    """
    A = np.asarray(A, np.float32)
    B = np.asarray(B, np.float32)
    if chan_exp is None:
        return A, B
    e = np.asarray(chan_exp, np.int64)
    As = np.ldexp(A.astype(np.float64), -e[None, :]).astype(np.float32)
    Bs = np.ldexp(B.astype(np.float64), e[:, None]).astype(np.float32)
    return As, Bs


def gemm_emulated(A, B, fmt=_split.FP16_S11, chan_exp=None):
    """Three-product compensated GEMM in float64 (no accumulation rounding)."""
    A, B = rescale_channels(A, B, chan_exp)
    Ah, Al, _, _ = _split.split(A, fmt)
    Bh, Bl, _, _ = _split.split(B, fmt)
    s = 1.0 / _split.LO_SCALE[fmt]
    return Ah @ Bh + s * (Ah @ Bl + Al @ Bh)


def truncation_term(A, B, fmt=_split.FP16_S11, chan_exp=None):
    """C_emul - C_ref written from the split residuals.

    With A = A1 + Ar, A1 = Ah + s Al (and likewise for B):
        A @ B = Ah Bh + s (Ah Bl + Al Bh) + s^2 Al Bl + A1 Br + Ar B
    so C_emul - C_ref = -(s^2 Al Bl + A1 Br + Ar B).
    """
    A, B = rescale_channels(A, B, chan_exp)
    Ah, Al, _, _ = _split.split(A, fmt)
    Bh, Bl, _, _ = _split.split(B, fmt)
    s = 1.0 / _split.LO_SCALE[fmt]
    A1 = Ah + s * Al
    B1 = Bh + s * Bl
    Ar = np.asarray(A, np.float64) - A1
    Br = np.asarray(B, np.float64) - B1
    return -(s * s * (Al @ Bl) + A1 @ Br + Ar @ np.asarray(B, np.float64))


def to_16bit(B, fmt=_split.FP16_S11):
    """B rounded to the format's 16-bit type (nearest even), returned as float64."""
    B = np.asarray(B, np.float32)
    if fmt == _split.FP16_S11:
        with np.errstate(over="ignore"):
            return _split.to_fp16(B).astype(np.float64)
    return _split.to_bf16_as_f32(B).astype(np.float64)


def gemm_two_product(A, W16, fmt=_split.FP16_S11, chan_exp=None):
    """Two-product compensated GEMM in float64: C = Ah W16 + s Al W16.

    The technical summary (section 2.B, "Mechanism") splits the input activations into a
    16-bit value and a residual and runs two 16-bit products whose results are added;
    the weights W16 are already 16-bit values (exactly representable), so they carry no
    residual.  With chan_exp, column k of A is scaled by 2^-e_k and row k of W16 by 2^e_k.
    """
    A = np.asarray(A, np.float32)
    W16 = np.asarray(W16, np.float64)
    if chan_exp is not None:
        e = np.asarray(chan_exp, np.int64)
        A = np.ldexp(A.astype(np.float64), -e[None, :]).astype(np.float32)
        W16 = np.ldexp(W16, e[:, None])
    Ah, Al, _, _ = _split.split(A, fmt)
    s = 1.0 / _split.LO_SCALE[fmt]
    return Ah @ W16 + s * (Al @ W16)


def two_product_truncation(A, W16, fmt=_split.FP16_S11):
    """gemm_two_product - A @ W16 = -Ar @ W16 with Ar = A - (Ah + s Al)."""
    Ah, Al, _, _ = _split.split(np.asarray(A, np.float32), fmt)
    s = 1.0 / _split.LO_SCALE[fmt]
    Ar = np.asarray(A, np.float32).astype(np.float64) - (Ah + s * Al)
    return -(Ar @ np.asarray(W16, np.float64))


def gemm_bf16_downcast(A, B):
    """BF16 inputs, FP32-exact products summed in float64, result stored as BF16."""
    Ab = _split.to_bf16_as_f32(A).astype(np.float64)
    Bb = _split.to_bf16_as_f32(B).astype(np.float64)
    C = (Ab @ Bb).astype(np.float32)
    return _split.to_bf16_as_f32(C).astype(np.float64)


def normwise_rel_err(C, C_ref):
    C = np.asarray(C, np.float64)
    C_ref = np.asarray(C_ref, np.float64)
    den = np.linalg.norm(C_ref)
    return float(np.linalg.norm(C - C_ref) / den) if den > 0 else float(np.linalg.norm(C))


def suggest_channel_exponents(A, limit=2.0 ** 14):
    """Exponent per K-channel that brings max|A[:, k]| to at most ``limit``.

    The pages only say that rare outlier channels are rescaled; this rule
    (e_k = ceil(log2(absmax_k / limit)) when absmax_k > limit, else 0) is a reading.
    """
    a = np.max(np.abs(np.asarray(A, np.float64)), axis=0)
    e = np.zeros(a.shape, np.int64)
    big = a > limit
    e[big] = np.ceil(np.log2(a[big] / limit)).astype(np.int64)
    return e.astype(np.int8)
