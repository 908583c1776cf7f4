"""Attention on INT16 Q/K/V (oracle; test infrastructure only).

Source: gist.science technical summary, section 2.A "Mitigating Attention Truncation
via INT16 Quantization", Mechanism: the INT16 tensor is unpacked into two FP16
tensors X_hi and X_lo whose combination carries more precision than one FP16.

The formula printed there, (X_hi + X_lo / 2**10), cannot be exact for INT16 data with
FP16 products summed over a 128-wide head (lo would span [0, 1023] and sum(lo*lo)
over 128 terms exceeds 2**24).  Reading used: a byte split,
    q = 256 * hi + lo,  hi = q >> 8 in [-128, 127],  lo = q & 255 in [0, 255],
both exactly representable in FP16.  The oracle's QK^T does not need the split at
all: it is the exact integer dot product in int64, which is what any exact
byte-split evaluation must reproduce.

Attention definition (no chunking, no online softmax, no FP32):
  hkv       = hq // (Hq / Hkv)                       (consecutive query heads share a KV head)
  pos_i     = kv_len[b] - Tq + i                     (queries are the last Tq positions)
  visible t : t < kv_len[b] and (not causal or t <= pos_i)
  logit_t   = S_int(q_i, k_t) * s_q * s_k[t] * softmax_scale      (float64)
  O_i       = sum_t softmax(logit)_t * s_v[t] * v_t               (float64)
  a query with no visible token (causal, position < 0, i.e. kv_len < Tq) has O_i = 0
  (the library's definition for that case; the pages do not reach it)

Parity: pinned (exhaustive byte-split reconstruction, int64 dots against Python
integers including extreme vectors, uniform-softmax and one-hot special cases,
single-token and causal-first-query cases).
"""
import numpy as np


def byte_split(q):
    """int16 -> (hi, lo) as int64 arrays with q == 256*hi + lo."""
    q = np.asarray(q, np.int64)
    return q >> 8, q & 255


def qk_int(q, k):
    """Exact integer dots: q [..., Tq, D] x k [..., T, D] -> int64 [..., Tq, T]."""
    q = np.asarray(q, np.int64)
    k = np.asarray(k, np.int64)
    return np.matmul(q, np.swapaxes(k, -1, -2))


def attention(q, q_scale, k_cache, k_scale, v_cache, v_scale, kv_len, softmax_scale,
              causal=False, return_s_int=False):
    """q [B,Hq,Tq,D] int16, q_scale [B,Hq,Tq]; caches [B,Hkv,Tmax,D] int16 with
    scales [B,Hkv,Tmax]; kv_len [B].  Returns O float64 [B,Hq,Tq,D] (and, if asked,
    the list of exact S_int blocks [Hq,Tq,kv_len[b]] per batch)."""
    q = np.asarray(q)
    B, Hq, Tq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, Tq, D), np.float64)
    s_blocks = []
    for b in range(B):
        L = int(kv_len[b])
        s_b = np.zeros((Hq, Tq, L), np.int64)
        for hq in range(Hq):
            hkv = hq // G
            S = qk_int(q[b, hq], k_cache[b, hkv, :L])  # [Tq, L]
            s_b[hq] = S
            logits = (S.astype(np.float64) * np.asarray(q_scale[b, hq], np.float64)[:, None]
                      * k_scale[b, hkv, :L].astype(np.float64)[None, :] * float(softmax_scale))
            if causal:
                pos = L - Tq + np.arange(Tq)
                mask = np.arange(L)[None, :] <= pos[:, None]
                logits = np.where(mask, logits, -np.inf)
            seen = np.isfinite(logits).any(axis=1) if L > 0 else np.zeros(Tq, bool)
            v = v_cache[b, hkv, :L].astype(np.float64) * v_scale[b, hkv, :L].astype(np.float64)[:, None]
            if seen.any():
                lg = logits[seen]
                m = np.max(lg, axis=1, keepdims=True)
                p = np.exp(lg - m)
                p /= np.sum(p, axis=1, keepdims=True)
                out[b, hq][seen] = p @ v
        s_blocks.append(s_b)
    return (out, s_blocks) if return_s_int else out

