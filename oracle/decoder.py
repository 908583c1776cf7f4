"""FP64 reference of the random-init decoder stack (oracle; test infrastructure only).

The pages evaluate HEAL-Full (INT16 Q/K/V plus compensated GEMMs) inside Llama/Qwen-class
decoders (gist.science technical summary, Results) and fix none of the block's details.
Readings used here (shared with the device harness only through this description):
  * Llama-style pre-norm block: h += W_o attn(rope(q), rope(k), v); h += W_down swiglu(W_gu x)
    with x = rmsnorm(h); RMSNorm weights 1, eps 1e-5; final RMSNorm then the LM head;
  * rotate-half RoPE: pairs (d, d + D/2), angle pos * theta^(-2d/D);
  * SwiGLU: silu(gate) * up with the gate in the first F columns of W_gu;
  * greedy decoding picks the lowest index among equal maxima;
  * Q, K (after RoPE) and V are quantized to INT16 per (token, head) exactly as in
    oracle.quant, from their values rounded to FP32; attention is oracle.attention.
Everything else is float64.  Teacher forcing: logits are evaluated on a given token
sequence (the device's), at chosen positions.

Parity: pinned (closed forms for RMSNorm, RoPE, SwiGLU, argmax; a stack with zeroed
layers reduces to the final norm and LM head; the block body on hand-built scatter weights,
written out element by element: one token at position 0, two layers in order, and two
tokens whose RoPE turn, INT16 rounding after RoPE and causal mask are each visible in the
logits).  The full stack's agreement with the device is a tolerance check, not a pin.
"""
import math

import numpy as np

from . import attention as OA
from . import quant as OQ


def rmsnorm(x, eps):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(x, pos, theta):
    """x [n, heads, D] float64, pos [n] -> rotated copy (rotate-half convention)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    half = D // 2
    inv = theta ** (-2.0 * np.arange(half) / D)
    ang = np.asarray(pos, np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def swiglu(gu, F):
    gu = np.asarray(gu, np.float64)
    g, u = gu[..., :F], gu[..., F:]
    return g / (1.0 + np.exp(-g)) * u


def argmax_lowest(x):
    return int(np.argmax(np.asarray(x)))   # numpy returns the first maximum


def _lm_head(x, W, chunk=16384):
    out = np.empty(W.shape[1], np.float64)
    for j in range(0, W.shape[1], chunk):
        out[j:j + chunk] = x @ W[:, j:j + chunk].astype(np.float64)
    return out


def decoder_logits(cfg, w, tokens, n_prompt, check):
    """Teacher-forced FP64 logits.

    cfg: synthetic.DecoderConfig; w: dict of float32 numpy arrays (synthetic.decoder_weights);
    tokens: the full token sequence (prompt followed by generated tokens); the prompt's
    n_prompt positions run as one causal block, later positions one at a time.
    check: positions whose next-token logits to return.  Returns {position: logits}.
    """
    H, Hq, Hkv, D, F = cfg.hidden, cfg.heads, cfg.kv_heads, cfg.head_dim, cfg.ffn
    last = max(check)
    T = last + 1
    kc = [np.zeros((1, Hkv, T, D), np.int16) for _ in range(cfg.layers)]
    ks = [np.zeros((1, Hkv, T), np.float32) for _ in range(cfg.layers)]
    vc = [np.zeros((1, Hkv, T, D), np.int16) for _ in range(cfg.layers)]
    vs = [np.zeros((1, Hkv, T), np.float32) for _ in range(cfg.layers)]
    out = {}
    blocks = [(0, n_prompt)] + [(p, p + 1) for p in range(n_prompt, T)]
    for (p0, p1) in blocks:
        if p0 > last:
            break
        n = p1 - p0
        h = w["embed"][np.asarray(tokens[p0:p1])].astype(np.float64)
        pos = np.arange(p0, p1)
        for l in range(cfg.layers):
            x = rmsnorm(h, cfg.eps)
            qkv = x @ w[f"wqkv{l}"].astype(np.float64)
            q = rope(qkv[:, :Hq * D].reshape(n, Hq, D), pos, cfg.rope_theta)
            k = rope(qkv[:, Hq * D:(Hq + Hkv) * D].reshape(n, Hkv, D), pos, cfg.rope_theta)
            v = qkv[:, (Hq + Hkv) * D:].reshape(n, Hkv, D)
            q16, qs = OQ.quantize_rows(q.astype(np.float32))            # [n, Hq, D], [n, Hq]
            k16, ksc = OQ.quantize_rows(k.astype(np.float32))
            v16, vsc = OQ.quantize_rows(v.astype(np.float32))
            kc[l][0, :, p0:p1] = k16.transpose(1, 0, 2)
            ks[l][0, :, p0:p1] = ksc.T
            vc[l][0, :, p0:p1] = v16.transpose(1, 0, 2)
            vs[l][0, :, p0:p1] = vsc.T
            qb = q16.transpose(1, 0, 2)[None]                          # [1, Hq, n, D]
            qsb = qs.T[None]                                           # [1, Hq, n]
            o = OA.attention(qb, qsb, kc[l][:, :, :p1], ks[l][:, :, :p1], vc[l][:, :, :p1], vs[l][:, :, :p1],
                             np.array([p1]), 1.0 / math.sqrt(D), causal=True)    # [1, Hq, n, D]
            attn = o[0].transpose(1, 0, 2).reshape(n, Hq * D)
            h = h + attn @ w[f"wo{l}"].astype(np.float64)
            x = rmsnorm(h, cfg.eps)
            act = swiglu(x @ w[f"wgu{l}"].astype(np.float64), F)
            h = h + act @ w[f"wdown{l}"].astype(np.float64)
        for p in range(p0, p1):
            if p in check:
                out[p] = _lm_head(rmsnorm(h[p - p0], cfg.eps), w["lm_head"])
    return out
