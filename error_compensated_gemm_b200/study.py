"""Reproducibility analogue and FP32-pipeline baseline on the random-init decoder stack.

The technical summary (Results) compares, on Llama/Qwen-class models held in 16-bit, a
native BF16 pipeline (every kernel stores its FP32 accumulator to BF16 memory: the boundary
truncation of its section 1), a full-FP32 pipeline (weights upcast, FP32 KV cache) and
HEAL-Full (INT16 Q/K/V plus compensated GEMMs), by answer flips against a reference and by
time per output token.  The same comparison here, on synthetic weights:

  * the weights are drawn as usual and rounded once so that every value is exactly
    representable in both BF16 and FP16 -- a 16-bit model, shared bit for bit by all
    pipelines, as the pages' models are;
  * FP64 (torch float64) is the truth and decodes greedily; FP32 (torch float32, TF32 off,
    FP32 KV cache), plain BF16 (torch bfloat16, every op storing 16 bits) and HEAL (this
    library's decoder, 16-bit weights, GEMMs in the two-product form of section 2.B with
    only the activations split, INT16 KV cache) are teacher-forced on its tokens;
  * per step: logits error and final-hidden MSE against FP64, argmax flips; each
    pipeline's own greedy decode gives the first free-running divergence;
  * time per output token: each pipeline's whole greedy decode captured once as a CUDA
    graph and replayed, so the ratios compare GPU work, not Python launch overhead.

The FP64, FP32 and BF16 pipelines are comparison arms written with torch's own ops (cuBLAS
GEMMs, scaled_dot_product_attention); they are not part of the library.
"""
import torch

from .decoder import Decoder


def sixteen_bit_weights(w):
    """Round every tensor to values exactly representable in both BF16 and FP16: BF16
    rounding first (8 significant bits), then FP16 (which keeps those bits in its normal
    range and rounds the few below 2^-17 onto its subnormal grid)."""
    out = {}
    for k, v in w.items():
        r = v.to(torch.bfloat16).to(torch.float32).to(torch.float16).to(torch.float32)
        assert torch.equal(r, r.to(torch.bfloat16).to(torch.float32)), k
        out[k] = r
    return out


class TorchDecoder:
    """The decoder block in plain torch ops at one precision (a comparison arm).  Every op
    reads and writes `dtype` tensors (for bf16: 16-bit stores at every kernel boundary); K
    and V are cached in `dtype`; attention is torch's scaled_dot_product_attention."""

    def __init__(self, cfg, w, dtype, dev, max_len):
        self.cfg, self.dtype, self.dev = cfg, dtype, dev
        self.w = {k: v.to(dev, dtype) for k, v in w.items()}
        half = cfg.head_dim // 2
        inv = torch.tensor([cfg.rope_theta ** (-2.0 * i / cfg.head_dim) for i in range(half)], dtype=torch.float64)
        ang = torch.arange(max_len, dtype=torch.float64)[:, None] * inv[None, :]
        self.cos, self.sin = torch.cos(ang).to(dev, dtype), torch.sin(ang).to(dev, dtype)
        shape = (max_len, cfg.kv_heads, cfg.head_dim)
        self.k = [torch.zeros(shape, dtype=dtype, device=dev) for _ in range(cfg.layers)]
        self.v = [torch.zeros(shape, dtype=dtype, device=dev) for _ in range(cfg.layers)]
        self.pos = 0

    def reset(self):
        self.pos = 0

    def _rms(self, x):
        return x * torch.rsqrt((x * x).mean(-1, keepdim=True) + self.cfg.eps)

    def _rope(self, x, p0):
        n, half = x.shape[0], self.cfg.head_dim // 2
        c, s = self.cos[p0:p0 + n, None, :], self.sin[p0:p0 + n, None, :]
        a, b = x[..., :half], x[..., half:]
        return torch.cat([a * c - b * s, b * c + a * s], dim=-1)

    def forward(self, ids):
        c = self.cfg
        F = torch.nn.functional
        n, p0 = ids.numel(), self.pos
        h = self.w["embed"][ids.long()]
        qd, kd = c.heads * c.head_dim, c.kv_heads * c.head_dim
        G = c.heads // c.kv_heads
        for l in range(c.layers):
            x = self._rms(h)
            qkv = x @ self.w[f"wqkv{l}"]
            q = self._rope(qkv[:, :qd].view(n, c.heads, c.head_dim), p0)
            k = self._rope(qkv[:, qd:qd + kd].view(n, c.kv_heads, c.head_dim), p0)
            self.k[l][p0:p0 + n] = k
            self.v[l][p0:p0 + n] = qkv[:, qd + kd:].view(n, c.kv_heads, c.head_dim)
            K = self.k[l][:p0 + n].repeat_interleave(G, dim=1).transpose(0, 1)   # [heads, T, D]
            V = self.v[l][:p0 + n].repeat_interleave(G, dim=1).transpose(0, 1)
            o = F.scaled_dot_product_attention(q.transpose(0, 1), K, V, is_causal=(n > 1 and p0 == 0),
                                               scale=c.head_dim ** -0.5)
            h = h + o.transpose(0, 1).reshape(n, qd) @ self.w[f"wo{l}"]
            x = self._rms(h)
            gu = x @ self.w[f"wgu{l}"]
            h = h + (F.silu(gu[:, :c.ffn]) * gu[:, c.ffn:]) @ self.w[f"wdown{l}"]
        self.pos = p0 + n
        self.last_hidden = self._rms(h[n - 1:n])
        return self.last_hidden @ self.w["lm_head"]

    def argmax_into(self, logits, out):
        out.copy_(torch.argmax(logits.float(), dim=-1).to(torch.int32).view(1))


class HealDecoder(Decoder):
    """The library's decoder with the comparison arms' interface."""

    def reset(self):
        self.pos_len = 0

    def argmax_into(self, logits, out):
        from . import _binding as H
        H.heal_argmax(logits, out)


def _teacher_forced(pipe, prompt, tokens, steps):
    pipe.reset()
    lg = pipe.forward(prompt)
    L, Hs = [], []
    for s in range(steps):
        L.append(lg.double().flatten())
        Hs.append(pipe.last_hidden.double().flatten())
        if s + 1 < steps:
            lg = pipe.forward(tokens[s:s + 1])
    return L, Hs


def _graph_decode(pipe, prompt, steps, dev):
    """Greedy decode after an eager prefill, all `steps` steps captured as one CUDA graph;
    returns (tokens, ms per output token of a replay)."""
    toks = torch.empty(steps, dtype=torch.int32, device=dev)
    pipe.reset()
    lg0 = pipe.forward(prompt)
    torch.cuda.synchronize(dev)
    cap = torch.cuda.Stream(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        lg = lg0
        for s in range(steps):
            pipe.argmax_into(lg, toks[s:s + 1])
            if s + 1 < steps:
                lg = pipe.forward(toks[s:s + 1])
    # the capture ran nothing: the caches still hold the prefill's state, which the graph
    # starts from (positions are fixed in the captured launches)
    g.replay()                                   # warm-up replay
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(dev)
    reps = 3
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    out = toks.clone()
    del g
    return out, e0.elapsed_time(e1) / reps / steps


def reproducibility_study(dev, cfg=None, prompt_len=512, steps=128, seed=10):
    """Runs the four pipelines; returns a JSON-ready dict (see the module docstring)."""
    import synthetic                      # the seeded input generators of the tests and the benchmark
    torch.backends.cuda.matmul.allow_tf32 = False
    torch.backends.cudnn.allow_tf32 = False
    max_len = prompt_len + steps + 64
    cfg = cfg or synthetic.DecoderConfig(max_pos=max_len)
    w = sixteen_bit_weights(synthetic.decoder_weights(cfg, seed=seed))
    prompt = synthetic.prompt_ids(prompt_len, cfg.vocab).to(dev)

    ref = TorchDecoder(cfg, w, torch.float64, dev, max_len)
    ref.reset()
    lg = ref.forward(prompt)
    L64, H64, T64 = [], [], []
    for s in range(steps):
        L64.append(lg.double().flatten())
        H64.append(ref.last_hidden.double().flatten())
        T64.append(int(torch.argmax(lg).item()))
        if s + 1 < steps:
            lg = ref.forward(torch.tensor([T64[-1]], dtype=torch.int32, device=dev))
    del ref
    torch.cuda.empty_cache()
    tokens = torch.tensor(T64, dtype=torch.int32, device=dev)
    top2 = [torch.topk(l, 2).values for l in L64]
    margins = [float(t[0] - t[1]) / float(l.abs().max()) for t, l in zip(top2, L64)]

    out = {"study": "reproducibility analogue: random-init decoder with 16-bit-representable weights, "
                    "teacher-forced on the FP64 greedy tokens; TPOT from one CUDA graph per greedy decode",
           "config": {"hidden": cfg.hidden, "heads": cfg.heads, "kv_heads": cfg.kv_heads,
                      "head_dim": cfg.head_dim, "ffn": cfg.ffn, "layers": cfg.layers, "vocab": cfg.vocab},
           "prompt": prompt_len, "steps": steps, "min_fp64_top2_margin": min(margins), "pipelines": {}}
    makers = {
        "fp32": lambda: TorchDecoder(cfg, w, torch.float32, dev, max_len),
        "bf16_downcast": lambda: TorchDecoder(cfg, w, torch.bfloat16, dev, max_len),
        "heal": lambda: HealDecoder(cfg, w, dev, max_len=max_len, weights16=True),
    }
    for name, make in makers.items():
        pipe = make()
        L, Hs = _teacher_forced(pipe, prompt, tokens, steps)
        rel = [float(torch.linalg.norm(a - b) / torch.linalg.norm(b)) for a, b in zip(L, L64)]
        mse = [float(((a - b) ** 2).mean()) for a, b in zip(Hs, H64)]
        flip_steps = [s for s, (a, b) in enumerate(zip(L, L64)) if int(torch.argmax(a)) != int(torch.argmax(b))]
        own, tpot = _graph_decode(pipe, prompt, steps, dev)
        own = own.tolist()
        first_div = next((i for i, (a, b) in enumerate(zip(own, T64)) if a != b), None)
        out["pipelines"][name] = {
            "logits_rel_err_mean": sum(rel) / len(rel), "logits_rel_err_max": max(rel),
            "final_hidden_mse_mean": sum(mse) / len(mse), "argmax_flips": len(flip_steps),
            "flip_steps": flip_steps[:16], "fp64_margin_at_flips": [margins[i] for i in flip_steps[:16]],
            "first_divergence_free_running": first_div, "tpot_ms": tpot}
        del pipe
        torch.cuda.empty_cache()
    b = out["pipelines"]["bf16_downcast"]["tpot_ms"]
    f = out["pipelines"]["fp32"]["tpot_ms"]
    for name, r in out["pipelines"].items():
        r["tpot_vs_bf16"] = r["tpot_ms"] / b
        r["tpot_vs_fp32"] = r["tpot_ms"] / f
    return out
