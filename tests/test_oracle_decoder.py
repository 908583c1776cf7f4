"""Pins for oracle.decoder (CPU only): closed forms of the glue and a degenerate stack."""
import math

import numpy as np
import pytest

import synthetic
from oracle import decoder as OD


def test_rmsnorm_constant_vector():
    x = np.full((2, 64), 3.0)
    x[1] = -0.5
    y = OD.rmsnorm(x, 1e-5)
    np.testing.assert_allclose(y[0], 3.0 / math.sqrt(9.0 + 1e-5), rtol=1e-15)
    np.testing.assert_allclose(y[1], -0.5 / math.sqrt(0.25 + 1e-5), rtol=1e-15)


def test_rope_hand_case_and_invariants():
    x = np.zeros((1, 1, 4))
    x[0, 0, 0] = 1.0
    y = OD.rope(x, [1], 10000.0)          # inv_freq = [1, 0.01]; pair (0, 2) turns by 1 radian
    np.testing.assert_allclose(y[0, 0], [math.cos(1.0), 0.0, math.sin(1.0), 0.0], atol=1e-15)
    rng = np.random.default_rng(0)
    z = rng.standard_normal((3, 2, 8))
    np.testing.assert_allclose(OD.rope(z, [0, 0, 0], 500000.0), z, rtol=0, atol=0)
    r = OD.rope(z, [5, 17, 300], 500000.0)
    np.testing.assert_allclose(r[..., :4] ** 2 + r[..., 4:] ** 2, z[..., :4] ** 2 + z[..., 4:] ** 2, rtol=1e-12)
    np.testing.assert_allclose(OD.rope(OD.rope(z, [2, 3, 4], 500000.0), [5, 6, 7], 500000.0),
                               OD.rope(z, [7, 9, 11], 500000.0), rtol=1e-12, atol=1e-12)


def test_swiglu_and_argmax():
    gu = np.array([[0.0, 1.0, 2.0, 3.0]])          # F = 2: gates (0, 1), ups (2, 3)
    np.testing.assert_allclose(OD.swiglu(gu, 2), [[0.0, 3.0 / (1.0 + math.exp(-1.0))]], rtol=1e-15)
    assert OD.argmax_lowest([1.0, 5.0, 2.0, 5.0]) == 1


def test_zeroed_layers_reduce_to_norm_and_head():
    cfg = synthetic.DecoderConfig(vocab=50, hidden=32, heads=4, kv_heads=2, head_dim=8, ffn=48, layers=2)
    w = {k: v.numpy() for k, v in synthetic.decoder_weights(cfg, seed=3).items()}
    for l in range(cfg.layers):
        w[f"wo{l}"][:] = 0
        w[f"wdown{l}"][:] = 0
    toks = [3, 7, 11, 2, 9]
    out = OD.decoder_logits(cfg, w, toks, n_prompt=3, check=[2, 4])
    for p in (2, 4):
        want = OD.rmsnorm(w["embed"][toks[p]].astype(np.float64), cfg.eps) @ w["lm_head"].astype(np.float64)
        np.testing.assert_allclose(out[p], want, rtol=1e-12)


def test_prompt_block_equals_one_token_at_a_time():
    """Running the prompt as one causal block gives the same logits as feeding its tokens
    one by one (the cache and the causal mask agree)."""
    cfg = synthetic.DecoderConfig(vocab=40, hidden=32, heads=4, kv_heads=2, head_dim=8, ffn=40, layers=2)
    w = {k: v.numpy() for k, v in synthetic.decoder_weights(cfg, seed=4).items()}
    toks = [1, 5, 9, 13, 17, 21]
    a = OD.decoder_logits(cfg, w, toks, n_prompt=6, check=[5])
    b = OD.decoder_logits(cfg, w, toks, n_prompt=1, check=[5])
    np.testing.assert_allclose(a[5], b[5], rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------------------------------
# The block body, pinned on hand-built weights.  Every weight matrix below is a scatter
# (each input index feeds one output index) so that the expected hidden state can be
# written element by element; each mistake a plausible misreading of the block would make
# -- V taken from the K columns, RoPE on V, quantizing before RoPE, the wrong GQA head
# mapping, a transposed projection, a missing or misplaced residual, a post-norm block, the
# SwiGLU gate and up halves swapped, no final norm -- moves at least one logit at O(1e-5)
# or more, far beyond the 1e-12 used here.
# ---------------------------------------------------------------------------------------

from oracle import quant as OQ


def _scatter(n_in, n_out, dst, scale=None):
    """Matrix W [n_in, n_out] with W[i, dst[i]] = scale[i] (1 by default): y = x @ W puts
    x[i] * scale[i] into y[dst[i]]."""
    W = np.zeros((n_in, n_out), np.float32)
    for i, j in enumerate(dst):
        W[i, j] = 1.0 if scale is None else scale[i]
    return W


def _rms(v):
    return [a / math.sqrt(sum(b * b for b in v) / len(v)) for a in v]   # eps = 0 in these configs


def _deq(row):
    """Dequantized INT16 row (per-row absmax code, as the decoder stores K and V)."""
    q, s = OQ.quantize_rows(np.asarray(row, np.float32)[None, None, :])
    return [float(c) * float(s[0, 0]) for c in q[0, 0]]


def _silu(g):
    return g / (1.0 + math.exp(-g))


def _single_token_block(e, wd, cfg):
    """Expected hidden state after one block for a one-token sequence at position 0
    (RoPE is the identity there and the softmax over one token is 1, so each query head
    returns the dequantized V of its KV head)."""
    Hq, Hkv, D, F = cfg.heads, cfg.kv_heads, cfg.head_dim, cfg.ffn
    x = _rms(e)
    v_cols = range((Hq + Hkv) * D, (Hq + 2 * Hkv) * D)
    v = [sum(x[i] * float(wd["wqkv"][i, c]) for i in range(len(x))) for c in v_cols]
    attn = []
    for hq in range(Hq):
        g = hq // (Hq // Hkv)                         # consecutive query heads share a KV head
        attn += _deq(v[g * D:(g + 1) * D])
    h = [e[j] + sum(attn[i] * float(wd["wo"][i, j]) for i in range(len(attn))) for j in range(len(e))]
    x2 = _rms(h)
    gu = [sum(x2[i] * float(wd["wgu"][i, c]) for i in range(len(x2))) for c in range(2 * F)]
    act = [_silu(gu[f]) * gu[F + f] for f in range(F)]
    return [h[j] + sum(act[f] * float(wd["wdown"][f, j]) for f in range(F)) for j in range(len(h))]


def _cfg8(layers):
    return synthetic.DecoderConfig(vocab=8, hidden=8, heads=4, kv_heads=2, head_dim=2, ffn=3, layers=layers,
                                   rope_theta=10000.0, eps=0.0)


def _layer8(seed, v_src, wo_dst, down_dst, gate_src, up_src):
    rng = np.random.default_rng(seed)
    wqkv = np.zeros((8, 16), np.float32)
    wqkv[:, :12] = rng.standard_normal((8, 12)).astype(np.float32)      # Q and K: any values
    for j, i in enumerate(v_src):                                        # V column 12 + j reads x[i]
        wqkv[i, 12 + j] = 1.0
    wgu = np.zeros((8, 6), np.float32)
    for f in range(3):
        wgu[gate_src[f], f] = 1.5                                        # gate f = 1.5 x[gate_src[f]]
        wgu[up_src[f], 3 + f] = -0.75                                    # up f = -0.75 x[up_src[f]]
    return {"wqkv": wqkv, "wo": _scatter(8, 8, wo_dst), "wgu": wgu,
            "wdown": _scatter(3, 8, down_dst, scale=[0.5, -2.0, 1.25])}


def test_block_single_token_closed_form():
    cfg = _cfg8(layers=1)
    s = [1.0, -1.0, 1.0, 1.0, -1.0, 1.0, -1.0, -1.0]
    e = [2.0 * a for a in s]                                             # rmsnorm(e) = s exactly
    L0 = _layer8(0, v_src=[5, 2, 7, 0], wo_dst=[3, 6, 0, 5, 1, 7, 2, 4], down_dst=[4, 1, 6],
                 gate_src=[0, 3, 6], up_src=[1, 4, 7])
    head_dst = [2, 7, 4, 0, 6, 1, 5, 3]
    w = {"embed": np.tile(np.asarray(e, np.float32), (cfg.vocab, 1)), "lm_head": _scatter(8, 8, head_dst)}
    w.update({f"{k}0": v for k, v in L0.items()})
    got = OD.decoder_logits(cfg, w, [3], n_prompt=1, check=[0])[0]
    h = _single_token_block(e, L0, cfg)
    y = _rms(h)
    want = [0.0] * 8
    for i, j in enumerate(head_dst):
        want[j] = y[i]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)
    # the V path is live: the attention output is about 1 per element, not zero
    assert max(abs(a - b) for a, b in zip(h, e)) > 0.5


def test_two_layers_chain_in_order():
    cfg = _cfg8(layers=2)
    e = [0.5, -1.5, 2.0, 0.25, -0.75, 1.0, -2.5, 0.125]
    L0 = _layer8(1, v_src=[1, 6, 3, 4], wo_dst=[5, 0, 7, 2, 6, 3, 1, 4], down_dst=[2, 5, 0],
                 gate_src=[7, 2, 5], up_src=[0, 3, 6])
    L1 = _layer8(2, v_src=[0, 7, 2, 5], wo_dst=[1, 4, 6, 0, 3, 7, 5, 2], down_dst=[6, 3, 1],
                 gate_src=[4, 1, 2], up_src=[5, 7, 0])
    w = {"embed": np.tile(np.asarray(e, np.float32), (cfg.vocab, 1)),
         "lm_head": np.eye(8, dtype=np.float32)}
    w.update({f"{k}0": v for k, v in L0.items()})
    w.update({f"{k}1": v for k, v in L1.items()})
    got = OD.decoder_logits(cfg, w, [0], n_prompt=1, check=[0])[0]
    # the embedding row passes through float32 storage, as the oracle reads it
    e32 = [float(np.float32(a)) for a in e]
    h = _single_token_block(_single_token_block(e32, L0, cfg), L1, cfg)
    np.testing.assert_allclose(got, _rms(h), rtol=1e-12, atol=1e-14)
    # the other order of the layers gives a different result
    h_swapped = _single_token_block(_single_token_block(e32, L1, cfg), L0, cfg)
    assert np.max(np.abs(np.asarray(_rms(h_swapped)) - got)) > 1e-3


def _rot(v, angle):
    c, s = math.cos(angle), math.sin(angle)
    return [v[0] * c - v[1] * s, v[1] * c + v[0] * s]


def test_two_token_block_rope_on_q_k_only_quantized_after_rope_and_causal():
    """Two prompt tokens at positions 0 and 1 with D = 2 (one RoPE pair, angle = position in
    radians).  Q = K = x and V = the swapped pair of x; output projection, LM head identity,
    MLP zero.  Expected: RoPE turns q and k (not v) by their position, then each row is
    quantized; position 0 sees only token 0 (causal), position 1 a softmax of two logits."""
    cfg = synthetic.DecoderConfig(vocab=2, hidden=2, heads=1, kv_heads=1, head_dim=2, ffn=1, layers=1,
                                  rope_theta=500000.0, eps=0.0)
    e = [[1.0, 1.0], [3.0 * math.cos(1.0), -3.0 * math.sin(1.0)]]
    wqkv = np.zeros((2, 6), np.float32)
    wqkv[0, 0] = wqkv[1, 1] = 1.0            # q = x
    wqkv[0, 2] = wqkv[1, 3] = 1.0            # k = x
    wqkv[1, 4] = wqkv[0, 5] = 1.0            # v = (x1, x0)
    w = {"embed": np.asarray(e, np.float32), "lm_head": np.eye(2, dtype=np.float32),
         "wqkv0": wqkv, "wo0": np.eye(2, dtype=np.float32),
         "wgu0": np.zeros((2, 2), np.float32), "wdown0": np.zeros((1, 2), np.float32)}
    got = OD.decoder_logits(cfg, w, [0, 1], n_prompt=2, check=[0, 1])

    e32 = [[float(np.float32(a)) for a in row] for row in e]
    x = [_rms(row) for row in e32]
    qk = [_rot(x[p], float(p)) for p in (0, 1)]                          # RoPE, then quantize
    codes, scales = OQ.quantize_rows(np.asarray(qk, np.float32)[:, None, :])
    codes = codes[:, 0].astype(np.int64)
    scales = scales[:, 0].astype(np.float64)
    v = [_deq([x[p][1], x[p][0]]) for p in (0, 1)]                       # V: no RoPE
    scale = 1.0 / math.sqrt(2.0)
    logit = lambda i, t: float(codes[i] @ codes[t]) * scales[i] * scales[t] * scale
    l10, l11 = logit(1, 0), logit(1, 1)
    m = max(l10, l11)
    p0, p1 = math.exp(l10 - m), math.exp(l11 - m)
    o1 = [(p0 * v[0][d] + p1 * v[1][d]) / (p0 + p1) for d in range(2)]
    o0 = v[0]                                                             # causal: token 0 only
    for p, o in ((0, o0), (1, o1)):
        want = _rms([e32[p][d] + o[d] for d in range(2)])
        np.testing.assert_allclose(got[p], want, rtol=1e-12, atol=1e-14)
    # the turned query at position 1 lies on the first axis, so its code row is exact
    assert list(codes[1]) == [32767, 0]


def test_swiglu_uses_gate_half_first():
    gu = np.array([[2.0, -1.0]])                                         # F = 1: gate 2, up -1
    got = OD.swiglu(gu, 1)[0, 0]
    assert got == pytest.approx(_silu(2.0) * -1.0, rel=1e-15)
    assert abs(got - _silu(-1.0) * 2.0) > 0.1
