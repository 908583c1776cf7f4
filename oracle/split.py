"""Hi/lo residual decomposition of FP32 operands (oracle; test infrastructure only).

Source: gist.science technical summary, section 2.B "Mitigating GEMM Truncation via
Algebraic Error Compensation" -- inputs are decomposed into a primary 16-bit value
and a residual error term; the overflow remark in the same section names FP16.

Readings (the pages name neither the 16-bit format nor a scale for the residual):
  * ``fp16_s11`` (default): hi = fp16_rn(x); lo = fp16_rn((x - hi) * 2**11).
    The residual is stored scaled by 2**11 so that it stays in FP16's normal range;
    the product terms that use it are scaled back by 2**-11.
  * ``bf16``: hi = bf16_rn(x); lo = bf16_rn(x - hi), unscaled.
  Rounding is round-to-nearest, ties-to-even, everywhere.

Parity: pinned (exhaustive mantissa sweeps against the exact nearest-value
definition, reconstruction bound, special values).
"""
import numpy as np
import torch

FP16_S11 = "fp16_s11"
BF16 = "bf16"
LO_SCALE = {FP16_S11: 2.0 ** 11, BF16: 1.0}


def to_fp16(x):
    """Round float32/float64 values to FP16, nearest-even (numpy's IEEE conversion)."""
    return np.asarray(x).astype(np.float16)


def to_bf16_as_f32(x):
    """Round float32 values to BF16, nearest-even; returned as float32 holding the BF16 value."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x_bf16_as_f32):
    """Upper 16 bits of a float32 that holds an exact BF16 value (its BF16 encoding)."""
    return (np.asarray(x_bf16_as_f32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def split(x, fmt=FP16_S11):
    """Split FP32 ``x`` into (hi, lo).

    Returns float64 arrays holding the exact 16-bit values, plus the raw 16-bit
    encodings (uint16) so that a bitwise comparison with a device split is possible:
    ``(hi, lo, hi_bits, lo_bits)``.  The residual x - hi is formed in float64, where
    it is exact.
    """
    x = np.asarray(x, dtype=np.float32)
    xd = x.astype(np.float64)
    if fmt == FP16_S11:
        with np.errstate(over="ignore"):
            hi16 = to_fp16(x)
        r = xd - hi16.astype(np.float64)
        with np.errstate(invalid="ignore", over="ignore"):
            lo16 = to_fp16(r * LO_SCALE[fmt])
        return (hi16.astype(np.float64), lo16.astype(np.float64),
                hi16.view(np.uint16), lo16.view(np.uint16))
    if fmt == BF16:
        hi = to_bf16_as_f32(x)
        r = (xd - hi.astype(np.float64)).astype(np.float32)  # exact: see module header
        lo = to_bf16_as_f32(r)
        return (hi.astype(np.float64), lo.astype(np.float64), bf16_bits(hi), bf16_bits(lo))
    raise ValueError(f"unknown split format {fmt!r}")


def reconstruct(hi, lo, fmt=FP16_S11):
    """hi + lo / scale in float64 (the value the compensated products see)."""
    return np.asarray(hi, np.float64) + np.asarray(lo, np.float64) / LO_SCALE[fmt]
