"""Seeded synthetic inputs shared by the tests, the benchmark and the CPU oracle.

This module holds no arithmetic of the method: it only draws random numbers
(PyTorch CPU generators, fixed seeds) in the shapes, distributions and outlier
structure of the paper's LLM workloads.  Outlier channels are a fixed set of
columns (about 1%) scaled by 20, echoing the remark in the gist.science technical
summary (section 2.B, "Overflow Handling") that outliers sit in under 1% of fixed
channels.

Workloads (sizes match the 8B-class decoder the paper evaluates):
  gemm_square   A[256x256], B[256x256] ~ N(0,1), both from seed 0
  gemm_prefill  X[M x K] ~ N(0,1) with 1% of columns x20 (seed 0, columns from
                randperm(seed+100)); W[K x N] ~ N(0, 0.02) (seed 1)
  gemm_decode   X[M x 4096] ~ N(0,1) (seed 0); W[4096 x 4096] ~ N(0, 0.02) (seed 1)
  kv_decode     K, V bf16 [B, T, Hkv, D] ~ N(0,1) with 1% of the Hkv*D flattened
                channels x20 (seeds 2 and 3); Q bf16 [B, Tq, Hq, D], 1% of Hq*D
                channels x20 (seed 4)
"""
import torch


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def normal(shape, seed=None, std=1.0, gen=None):
    g = gen if gen is not None else _gen(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def outlier_columns(n_cols, frac, seed):
    """Fixed outlier column indices: the first round(frac*n_cols) of randperm(seed+100)."""
    k = max(1, int(round(frac * n_cols)))
    return torch.randperm(n_cols, generator=_gen(seed + 100))[:k]


def with_outliers(x, frac, factor, seed):
    """Scale a fixed ~frac of the last-axis channels of x (viewed as [..., C]) by factor."""
    cols = outlier_columns(x.shape[-1], frac, seed)
    x[..., cols] *= factor
    return x


def gemm_square(n=256, seed=0):
    g = _gen(seed)
    A = torch.randn(n, n, generator=g, dtype=torch.float32)
    B = torch.randn(n, n, generator=g, dtype=torch.float32)
    return A, B


def gemm_prefill(M=4096, K=4096, N=14336, seed_x=0, seed_w=1, outlier_frac=0.01, factor=20.0):
    X = with_outliers(normal((M, K), seed_x), outlier_frac, factor, seed_x)
    W = normal((K, N), seed_w, std=0.02)
    return X, W


def gemm_decode(M, K=4096, N=4096, seed_x=0, seed_w=1):
    return normal((M, K), seed_x), normal((K, N), seed_w, std=0.02)


def kv_decode(B=8, T=8192, Hkv=8, Hq=32, D=128, Tq=1, seeds=(2, 3, 4), outlier_frac=0.01, factor=20.0):
    """Returns (Q, K, V) as bf16 CPU tensors shaped [B, Tq, Hq, D], [B, T, Hkv, D] x2."""
    out = []
    for (shape, seed) in (((B, T, Hkv, D), seeds[0]), ((B, T, Hkv, D), seeds[1])):
        x = normal(shape, seed).view(B, T, Hkv * D)
        with_outliers(x, outlier_frac, factor, seed)
        out.append(x.view(shape).to(torch.bfloat16))
    q = normal((B, Tq, Hq, D), seeds[2]).view(B, Tq, Hq * D)
    with_outliers(q, outlier_frac, factor, seeds[2])
    K_, V_ = out
    return q.view(B, Tq, Hq, D).to(torch.bfloat16), K_, V_


def rand_int16(shape, seed, lo=-32767, hi=32767):
    return torch.randint(lo, hi + 1, shape, generator=_gen(seed), dtype=torch.int32).to(torch.int16)


class DecoderConfig:
    """Shape of the random-init decoder stack (8B-class Llama-style block by default)."""

    def __init__(self, vocab=128256, hidden=4096, heads=32, kv_heads=8, head_dim=128, ffn=14336, layers=2,
                 rope_theta=500000.0, eps=1e-5, max_pos=1024):
        self.vocab, self.hidden, self.heads, self.kv_heads = vocab, hidden, heads, kv_heads
        self.head_dim, self.ffn, self.layers = head_dim, ffn, layers
        self.rope_theta, self.eps, self.max_pos = rope_theta, eps, max_pos

    @property
    def qkv_dim(self):
        return (self.heads + 2 * self.kv_heads) * self.head_dim


def decoder_weights(cfg, seed=10):
    """FP32 CPU tensors: embedding [vocab, H] ~ N(0,1); per layer wqkv [H, (Hq+2Hkv)D],
    wo [Hq*D, H], w_gate_up [H, 2F] (gate columns first), w_down [F, H]; lm_head [H, vocab];
    every linear ~ N(0, 0.02).  RMSNorm weights are 1 and not stored."""
    H = cfg.hidden
    w = {"embed": normal((cfg.vocab, H), seed)}
    for l in range(cfg.layers):
        s = seed + 1 + 10 * l
        w[f"wqkv{l}"] = normal((H, cfg.qkv_dim), s, std=0.02)
        w[f"wo{l}"] = normal((cfg.heads * cfg.head_dim, H), s + 1, std=0.02)
        w[f"wgu{l}"] = normal((H, 2 * cfg.ffn), s + 2, std=0.02)
        w[f"wdown{l}"] = normal((cfg.ffn, H), s + 3, std=0.02)
    w["lm_head"] = normal((H, cfg.vocab), seed + 9, std=0.02)
    return w


def prompt_ids(n, vocab, seed=5):
    """Uniform random token ids (int32)."""
    return torch.randint(0, vocab, (n,), generator=_gen(seed), dtype=torch.int32)
