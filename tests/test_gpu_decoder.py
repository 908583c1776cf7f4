"""GPU tests of the decoder glue kernels and the 2-layer random-init decoder stack.

Logits are compared with the teacher-forced FP64 oracle (oracle.decoder) on the device's
own token sequence.  Tolerance (normwise relative, per checked position): the stack is a
chain of about 8 compensated GEMMs (each <= 1e-6, measured ~2e-7), INT16 quantizations whose
codes can move by one step when their FP32 inputs differ in the last bits (one step is
2^-15 of the row's absmax), FP32 glue (RMSNorm, RoPE, SwiGLU: a few ulp each) and the FP32
softmax (see tests/test_gpu_attention.py).  Bound used: 1e-4, with the measured value printed.
Greedy tokens must agree with the oracle wherever the oracle's top-2 logit margin exceeds
1e-3 * ||logits||_inf (a gap far larger than the error bound).
"""
import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
import synthetic
from error_compensated_gemm_b200.decoder import Decoder, rope_tables
from oracle import decoder as OD
from tests.gpu_helpers import dev, status_ok, to_np

pytestmark = pytest.mark.gpu
TOL_LOGITS = 1e-4


def test_glue_kernels_against_oracle():
    d = dev()
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 4096)).astype(np.float32) * 3
    y = torch.empty(5, 4096, device=d)
    heal.heal_rmsnorm(torch.from_numpy(x).to(d), None, y, 1e-5)
    np.testing.assert_allclose(to_np(y), OD.rmsnorm(x, 1e-5), rtol=2e-6, atol=2e-6)

    q = rng.standard_normal((7, 32 * 128)).astype(np.float32)
    pos = np.array([0, 1, 5, 100, 511, 700, 1023], np.int32)
    cos, sin = rope_tables(1024, 128, 500000.0)
    qd = torch.from_numpy(q).to(d)
    heal.heal_rope(qd, 32, 128, torch.from_numpy(pos).to(d), cos.to(d), sin.to(d))
    want = OD.rope(q.reshape(7, 32, 128), pos, 500000.0).reshape(7, -1)
    np.testing.assert_allclose(to_np(qd), want, rtol=1e-5, atol=1e-5)

    gu = rng.standard_normal((3, 2 * 1000)).astype(np.float32) * 4
    out = torch.empty(3, 1000, device=d)
    heal.heal_swiglu(torch.from_numpy(gu).to(d), out)
    np.testing.assert_allclose(to_np(out), OD.swiglu(gu, 1000), rtol=1e-6, atol=1e-6)

    a = rng.standard_normal(10001).astype(np.float32)
    b = rng.standard_normal(10001).astype(np.float32)
    ad = torch.from_numpy(a).to(d)
    heal.heal_add(ad, torch.from_numpy(b).to(d))
    np.testing.assert_array_equal(to_np(ad), a + b)

    logits = rng.standard_normal((3, 128256)).astype(np.float32)
    logits[1, 77] = logits[1, 5000] = 50.0            # tie: lowest index wins
    idx = torch.empty(3, dtype=torch.int32, device=d)
    heal.heal_argmax(torch.from_numpy(logits).to(d), idx)
    assert list(to_np(idx)) == [OD.argmax_lowest(r) for r in logits] and to_np(idx)[1] == 77

    table = rng.standard_normal((100, 64)).astype(np.float32)
    ids = np.array([5, 0, 99, 42], np.int32)
    emb = torch.empty(4, 64, device=d)
    heal.heal_embedding_gather(torch.from_numpy(table).to(d), torch.from_numpy(ids).to(d), emb)
    status_ok()
    np.testing.assert_array_equal(to_np(emb), table[ids])
    heal.heal_embedding_gather(torch.from_numpy(table).to(d), torch.tensor([3, 100], dtype=torch.int32, device=d),
                               emb[:2])
    torch.cuda.synchronize()
    assert heal.heal_get_device_status() == heal.HEAL_ERR_INVALID_ARGUMENT
    assert heal.heal_get_device_status() == heal.HEAL_OK          # the flag is cleared
    np.testing.assert_array_equal(to_np(emb[1]), 0)


def _check_against_oracle(cfg, w, prompt, tokens, logits, check):
    seq = list(prompt.numpy()) + list(tokens)
    ref = OD.decoder_logits(cfg, {k: v.numpy() for k, v in w.items()}, seq, len(prompt), check)
    n0 = len(prompt) - 1
    errs = []
    for p in check:
        got = to_np(logits[p - n0][0]).astype(np.float64)
        r = ref[p]
        err = np.linalg.norm(got - r) / np.linalg.norm(r)
        errs.append(err)
        assert err <= TOL_LOGITS, (p, err)
        top2 = np.sort(r)[-2:]
        if top2[1] - top2[0] > 1e-3 * np.max(np.abs(r)) and p - n0 < len(tokens):
            assert tokens[p - n0] == OD.argmax_lowest(r), p
    return errs


def test_tiny_decoder_every_position():
    d = dev()
    cfg = synthetic.DecoderConfig(vocab=1000, hidden=256, heads=4, kv_heads=1, head_dim=64, ffn=512, layers=2,
                                  max_pos=64)
    w = synthetic.decoder_weights(cfg, seed=21)
    prompt = synthetic.prompt_ids(32, cfg.vocab, seed=6)
    dec = Decoder(cfg, w, d, max_len=64)
    toks, logits = dec.generate(prompt, 8)
    status_ok()
    toks = list(to_np(toks))
    errs = _check_against_oracle(cfg, w, prompt, toks, logits, check=list(range(31, 31 + 8)))
    print("tiny decoder logit errors", max(errs))


@pytest.mark.slow
def test_config5_decoder_bitwise_and_oracle():
    """hidden 4096, 32/8 heads, head_dim 128, FFN 14336, vocab 128256, 2 layers; 512-token
    random-id prompt, 128 greedy steps; two runs must agree bit for bit."""
    d = dev()
    cfg = synthetic.DecoderConfig(max_pos=704)
    w = synthetic.decoder_weights(cfg)
    prompt = synthetic.prompt_ids(512, cfg.vocab, seed=5)
    dec = Decoder(cfg, w, d, max_len=704)
    t1, l1 = dec.generate(prompt, 128)
    t2, l2 = dec.generate(prompt, 128)
    status_ok()
    assert torch.equal(t1, t2)
    for a, b in zip(l1, l2):
        assert torch.equal(a, b)
    errs = _check_against_oracle(cfg, w, prompt, list(to_np(t1)), l1, check=[511, 512, 513])
    print("config-5 logit errors", errs)


def test_heads_to_rows_is_an_exact_transpose():
    d = dev()
    g = torch.Generator().manual_seed(21)
    for (B, Hh, T, D) in ((1, 32, 515, 128), (2, 3, 7, 64), (1, 1, 1, 4)):
        x = torch.randn(B, Hh, T, D, generator=g)
        y = torch.full((B, T, Hh, D), float("nan"), device=d)
        heal.heal_heads_to_rows(x.to(d), y)
        status_ok()
        assert torch.equal(to_np_t(y), x.permute(0, 2, 1, 3))


def to_np_t(t):
    return t.detach().cpu()


def test_argmax_vector_and_scalar_paths():
    """The argmax kernel reads 16-byte vectors when a row is 16-byte aligned (n % 4 == 0) and
    single values otherwise; both give numpy's first maximum, on ties, a lone finite value
    among -inf, and maxima at the first and the last index (the ragged tail)."""
    d = torch.device("cuda:0")
    rng = np.random.default_rng(7)
    for n in (128256, 10001, 4, 3):
        x = rng.standard_normal((5, n)).astype(np.float32)
        x[1, n // 3] = x[1, n - 1] = 60.0
        x[2, :] = -np.inf
        x[2, n - 1] = -1e38
        x[3, 0] = 70.0
        x[4, n - 1] = 80.0
        idx = torch.empty(5, dtype=torch.int32, device=d)
        heal.heal_argmax(torch.from_numpy(x).to(d), idx)
        assert list(idx.cpu().numpy()) == [OD.argmax_lowest(r) for r in x], n
