"""A random-init Llama-style decoder stack run entirely through libheal.so.

Every linear layer is the error-compensated GEMM (FP32 in, FP32 out), Q/K/V go through the
INT16 quantizer into an INT16 KV cache, attention is the INT16 attention kernel, and the
glue (embedding, RMSNorm, RoPE, SwiGLU, residual, argmax) is the library's FP32 kernels:
the "HEAL-Full" pipeline of the gist.science technical summary (Results), on synthetic
weights.  PyTorch only allocates buffers and supplies the stream.

Prefill runs the projections, the MLP and causal attention on all prompt rows at once
(M = prompt length; attention through the library's prefill kernel, queries at positions
p0 .. p0+n-1 of a context of p0+n tokens).  That kernel is built for head_dim 128; other
head sizes run prefill attention one query position at a time with the decode kernel.
"""
import math

import torch

from . import _binding as H


def rope_tables(max_pos, head_dim, theta):
    """FP32 cos/sin tables [max_pos, head_dim/2], evaluated in float64 on the host."""
    half = head_dim // 2
    inv = torch.tensor([theta ** (-2.0 * i / head_dim) for i in range(half)], dtype=torch.float64)
    ang = torch.arange(max_pos, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cos(ang).float(), torch.sin(ang).float()


_LINEARS = ("wqkv", "wo", "wgu", "wdown")


class Decoder:
    def __init__(self, cfg, weights, device, max_len=None, presplit_weights=True, weights16=False):
        """presplit_weights: split every linear weight once into its 16-bit hi and lo parts
        (heal_split, the same encodings the GEMM kernels produce) and keep only those; the
        GEMMs then split only the activations.  The results are the same bits either way.
        weights16: hold every linear weight as FP16 values instead (the weights must be
        FP16-representable, as a 16-bit model's are; converting others rounds them): every
        GEMM is then the two-product form, Ah.W + 2^-11 Al.W with only the activations split
        (technical summary, section 2.B), and streams half the weight bytes."""
        self.cfg = c = cfg
        self.dev = device
        self.max_len = max_len or c.max_pos
        self.w = {k: v.to(device).contiguous() for k, v in weights.items()}
        self.parts = {}
        self.w16 = {}
        if weights16:
            for k in [f"{n}{l}" for l in range(c.layers) for n in _LINEARS] + ["lm_head"]:
                self.w16[k] = self.w[k].half()
                self.w[k] = None
        elif presplit_weights:
            names = [f"{n}{l}" for l in range(c.layers) for n in _LINEARS] + ["lm_head"]
            for k in names:
                w = self.w[k]
                hi = torch.empty(w.shape, dtype=torch.int16, device=device)
                lo = torch.empty(w.shape, dtype=torch.int16, device=device)
                H.heal_split(w, hi, lo)
                self.parts[k] = (hi, lo)
                self.w[k] = None             # the FP32 copy is not needed any more
            torch.cuda.synchronize(device)
        cos, sin = rope_tables(self.max_len, c.head_dim, c.rope_theta)
        self.cos, self.sin = cos.to(device), sin.to(device)
        f32, i16 = torch.float32, torch.int16
        Tmax = (self.max_len + 63) // 64 * 64
        self.Tmax = Tmax
        self.kc = [torch.zeros(1, c.kv_heads, Tmax, c.head_dim, dtype=i16, device=device) for _ in range(c.layers)]
        self.ks = [torch.zeros(1, c.kv_heads, Tmax, dtype=f32, device=device) for _ in range(c.layers)]
        self.vc = [torch.zeros(1, c.kv_heads, Tmax, c.head_dim, dtype=i16, device=device) for _ in range(c.layers)]
        self.vs = [torch.zeros(1, c.kv_heads, Tmax, dtype=f32, device=device) for _ in range(c.layers)]
        shapes = [(1, c.qkv_dim, c.hidden), (1, c.hidden, c.heads * c.head_dim), (1, 2 * c.ffn, c.hidden),
                  (1, c.hidden, c.ffn), (1, c.vocab, c.hidden)]
        ws = max(H.heal_gemm_workspace_bytes(m, n, k) for (m, n, k) in shapes)
        self.gemm_ws = torch.empty(max(1, ws // 4), dtype=f32, device=device)
        self.attn_ws = torch.empty(max(H.heal_attention_workspace_bytes_gqa(1, c.heads, c.kv_heads, q, Tmax)
                                       for q in (1, self.max_len)) // 4, dtype=f32, device=device)
        self.kv_len = torch.arange(1, Tmax + 1, dtype=torch.int32, device=device)   # kv_len for position t: t + 1
        self.positions = torch.arange(0, Tmax, dtype=torch.int32, device=device)
        self.pos_len = 0
        self.rms_w = None

    # ---- building blocks (each one library call) ----
    def _linear(self, x, key, out):
        if key in self.w16:
            H.heal_gemm_compensated(x, self.w16[key], out, b_16bit=True, workspace=self.gemm_ws, b_static=True)
        elif key in self.parts:
            hi, lo = self.parts[key]
            H.heal_gemm_compensated(x, hi, out, b_lo=lo, workspace=self.gemm_ws, b_static=True)
        else:
            H.heal_gemm_compensated(x, self.w[key], out, workspace=self.gemm_ws)

    def _layer(self, l, h, n, p0):
        c = self.cfg
        d = self.dev
        x = torch.empty_like(h)
        H.heal_rmsnorm(h, self.rms_w, x, c.eps)
        qkv = torch.empty(n, c.qkv_dim, device=d)
        self._linear(x, f"wqkv{l}", qkv)
        pos = self.positions[p0:p0 + n]
        qd = c.heads * c.head_dim
        H.heal_rope(qkv, c.heads, c.head_dim, pos, self.cos, self.sin)                 # q heads
        H.heal_rope(qkv[:, qd:], c.kv_heads, c.head_dim, pos, self.cos, self.sin)      # k heads (in place)
        # INT16 Q (all rows in one call: [1, Hq, n, D]; one position a call: [n, Hq, 1, D]),
        # K/V into the layer's cache at positions p0 .. p0+n-1
        one_call = n == 1 or c.head_dim == 128
        R, D = c.qkv_dim, c.head_dim
        kd = c.kv_heads * D
        if one_call:
            q16 = torch.empty(1, c.heads, n, D, dtype=torch.int16, device=d)
            qsc = torch.empty(1, c.heads, n, device=d)
            H.heal_kv_quantize_int16(qkv.as_strided((1, n, c.heads, D), (n * R, R, D, 1), qkv.storage_offset()),
                                     q16, qsc)
        else:
            q16 = torch.empty(n, c.heads, 1, D, dtype=torch.int16, device=d)
            qsc = torch.empty(n, c.heads, 1, device=d)
            H.heal_kv_quantize_int16(qkv.as_strided((n, 1, c.heads, D), (R, R, D, 1), qkv.storage_offset()),
                                     q16, qsc)
        H.heal_kv_quantize_int16(qkv.as_strided((1, n, c.kv_heads, D), (n * R, R, D, 1), qkv.storage_offset() + qd),
                                 self.kc[l], self.ks[l], t_offset=p0)
        H.heal_kv_quantize_int16(qkv.as_strided((1, n, c.kv_heads, D), (n * R, R, D, 1),
                                                qkv.storage_offset() + qd + kd),
                                 self.vc[l], self.vs[l], t_offset=p0)
        scale = 1.0 / math.sqrt(c.head_dim)
        if not one_call:
            attn = torch.empty(n, c.heads * D, device=d)
            for i in range(n):
                t = p0 + i
                H.heal_attention_int16(q16[i:i + 1], qsc[i:i + 1], self.kc[l], self.ks[l], self.vc[l], self.vs[l],
                                       self.kv_len[t:t + 1], scale, attn[i:i + 1].view(1, c.heads, 1, D),
                                       self.attn_ws)
        elif n == 1:
            attn = torch.empty(1, c.heads * D, device=d)
            H.heal_attention_int16(q16, qsc, self.kc[l], self.ks[l], self.vc[l], self.vs[l],
                                   self.kv_len[p0:p0 + 1], scale, attn.view(1, c.heads, 1, D), self.attn_ws)
        else:
            attn_h = torch.empty(1, c.heads, n, D, device=d)
            H.heal_attention_int16(q16, qsc, self.kc[l], self.ks[l], self.vc[l], self.vs[l],
                                   self.kv_len[p0 + n - 1:p0 + n], scale, attn_h, self.attn_ws, causal=True)
            attn = torch.empty(n, c.heads * D, device=d)
            H.heal_heads_to_rows(attn_h, attn.view(1, n, c.heads, D))
        o = torch.empty(n, c.hidden, device=d)
        self._linear(attn, f"wo{l}", o)
        H.heal_add(h, o)
        H.heal_rmsnorm(h, self.rms_w, x, c.eps)
        gu = torch.empty(n, 2 * c.ffn, device=d)
        self._linear(x, f"wgu{l}", gu)
        act = torch.empty(n, c.ffn, device=d)
        H.heal_swiglu(gu, act)
        dn = torch.empty(n, c.hidden, device=d)
        self._linear(act, f"wdown{l}", dn)
        H.heal_add(h, dn)

    def forward(self, ids):
        """Run len(ids) new positions; returns FP32 logits of the last one [1, vocab]."""
        c = self.cfg
        n = ids.numel()
        p0 = self.pos_len
        if p0 + n > self.max_len:
            raise ValueError("sequence longer than the cache")
        h = torch.empty(n, c.hidden, device=self.dev)
        H.heal_embedding_gather(self.w["embed"], ids, h)
        for l in range(c.layers):
            self._layer(l, h, n, p0)
        self.pos_len = p0 + n
        x = torch.empty(1, c.hidden, device=self.dev)
        H.heal_rmsnorm(h[n - 1:n], self.rms_w, x, c.eps)
        self.last_hidden = x                     # final normed hidden state of the last position
        logits = torch.empty(1, c.vocab, device=self.dev)
        self._linear(x, "lm_head", logits)
        return logits

    def generate(self, prompt, steps):
        """Greedy decoding: returns (tokens [steps] int32 on the device, list of logits per step
        including the prefill's last position)."""
        self.pos_len = 0
        ids = prompt.to(self.dev)
        out = torch.empty(steps, dtype=torch.int32, device=self.dev)
        logits = self.forward(ids)
        all_logits = [logits]
        for s in range(steps):
            H.heal_argmax(logits, out[s:s + 1].view(1))
            if s + 1 < steps:
                logits = self.forward(out[s:s + 1])
                all_logits.append(logits)
        return out, all_logits
