"""Per-token, per-head symmetric INT16 quantization (oracle; test infrastructure only).

Source: gist.science technical summary, section 2.A "Mitigating Attention Truncation
via INT16 Quantization" -- Q, K and V are stored as INT16, keeping the KV cache at a
16-bit footprint.  The authors' v2 abstract states the same mechanism.

The pages give neither the granularity nor the rounding.  Readings used:
  * one scale per (token, head) row of ``head_dim`` values, symmetric, range
    [-32767, 32767] (-32768 unused);
  * all decisions in FP32, as a device kernel takes them:
        absmax = max |x|             (exact)
        inv    = fp32(32767 / absmax)
        q      = clamp(rint_half_even(fp32(x * inv)), -32767, 32767)
        s      = fp32(absmax / 32767)
    and absmax == 0 gives s = 0, q = 0.
  * inputs given in BF16 are widened to FP32 exactly first.

Parity: pinned (hand-worked values at power-of-two absmax, the round-trip bound
|x - q s| <= s/2 + 2**-22 absmax, zero and constant rows, absmax -> +-32767).
"""
import numpy as np

QMAX = 32767


def quantize_rows(x):
    """Quantize the last axis of float32 ``x``; returns (q int16, s float32[...])."""
    x = np.asarray(x, np.float32)
    absmax = np.max(np.abs(x), axis=-1)
    nz = absmax > 0
    safe = np.where(nz, absmax, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(QMAX) / safe).astype(np.float32)
    y = (x * inv[..., None]).astype(np.float32)
    q = np.clip(np.rint(y), -QMAX, QMAX)
    q = np.where(nz[..., None], q, 0).astype(np.int16)
    s = np.where(nz, (absmax / np.float32(QMAX)).astype(np.float32), np.float32(0)).astype(np.float32)
    return q, s


def quantize_kv(x):
    """[B, T, H, D] float32 -> cache layout q [B, H, T, D] int16, s [B, H, T] float32."""
    x = np.asarray(x, np.float32)
    q, s = quantize_rows(x)
    return np.ascontiguousarray(q.transpose(0, 2, 1, 3)), np.ascontiguousarray(s.transpose(0, 2, 1))


def dequantize(q, s):
    """q * s in float64 (the values the attention definition uses)."""
    return np.asarray(q, np.float64) * np.asarray(s, np.float64)[..., None]
