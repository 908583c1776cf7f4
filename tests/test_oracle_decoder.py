"""Pins for oracle.decoder (CPU only): closed forms of the glue and a degenerate stack."""
import math

import numpy as np

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
