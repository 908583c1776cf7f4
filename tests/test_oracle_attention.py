"""Pins for oracle.attention (CPU only).

gist.science technical summary, section 2.A: INT16 Q/K/V unpacked into two FP16
tensors for the attention contractions.  Read as the byte split q = 256*hi + lo.
"""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import quant as Q


def test_byte_split_all_int16_values():
    q = np.arange(-32768, 32768, dtype=np.int64).astype(np.int16)
    hi, lo = A.byte_split(q)
    np.testing.assert_array_equal(256 * hi + lo, q.astype(np.int64))
    assert hi.min() == -128 and hi.max() == 127 and lo.min() == 0 and lo.max() == 255
    assert tuple(x[32768 - 32767] for x in (hi, lo)) == (-128, 1)   # q = -32767
    # both parts are integers of at most 8 significant bits: exact in FP16
    assert np.all(hi.astype(np.float16).astype(np.int64) == hi)
    assert np.all(lo.astype(np.float16).astype(np.int64) == lo)


@pytest.mark.parametrize("case", ["max", "min", "mixed", "alt", "one_big"])
def test_byte_split_partial_sums_stay_exact_in_fp32_at_d128(case):
    D = 128
    if case == "max":
        q = np.full(D, 32767); k = np.full(D, 32767)
    elif case == "min":
        q = np.full(D, -32767); k = np.full(D, -32767)
    elif case == "mixed":
        q = np.full(D, -32767); k = np.full(D, 32767)
    elif case == "alt":
        q = np.where(np.arange(D) % 2 == 0, 32767, -32768); k = np.where(np.arange(D) % 3 == 0, 255, -1)
    else:
        q = np.ones(D, np.int64); k = np.ones(D, np.int64); q[7] = 32767; k[7] = -32768
    q = q.astype(np.int64); k = k.astype(np.int64)
    qh, ql = A.byte_split(q.astype(np.int16))
    kh, kl = A.byte_split(k.astype(np.int16))
    s_hh = int(np.dot(qh, kh)); s_x = int(np.dot(qh, kl) + np.dot(ql, kh)); s_ll = int(np.dot(ql, kl))
    for part in (s_hh, s_x, s_ll):
        assert abs(part) < 2 ** 24                     # every FP32 partial sum is an exact integer
    exact = sum(int(a) * int(b) for a, b in zip(q, k))
    assert 65536 * s_hh + 256 * s_x + s_ll == exact
    assert int(A.qk_int(q[None, :].astype(np.int16), k[None, :].astype(np.int16))[0, 0]) == exact


def test_qk_int_matches_python_integers():
    rng = np.random.default_rng(1)
    q = rng.integers(-32767, 32768, size=(3, 128)).astype(np.int16)
    k = rng.integers(-32767, 32768, size=(17, 128)).astype(np.int16)
    S = A.qk_int(q, k)
    for i in range(3):
        for j in range(17):
            assert int(S[i, j]) == sum(int(a) * int(b) for a, b in zip(q[i], k[j]))
    assert np.abs(S).max() > 2 ** 31                   # needs more than 32 bits: int64 is required


def _tiny_case(seed, B=1, Hq=4, Hkv=2, Tq=1, Tmax=6, D=8):
    rng = np.random.default_rng(seed)
    q = rng.integers(-300, 300, size=(B, Hq, Tq, D)).astype(np.int16)
    k = rng.integers(-300, 300, size=(B, Hkv, Tmax, D)).astype(np.int16)
    v = rng.integers(-32767, 32768, size=(B, Hkv, Tmax, D)).astype(np.int16)
    qs = rng.uniform(1e-3, 2e-3, size=(B, Hq, Tq)).astype(np.float32)
    ks = rng.uniform(1e-3, 2e-3, size=(B, Hkv, Tmax)).astype(np.float32)
    vs = rng.uniform(1e-4, 2e-4, size=(B, Hkv, Tmax)).astype(np.float32)
    return q, qs, k, ks, v, vs


def test_attention_against_scalar_python_loop():
    q, qs, k, ks, v, vs = _tiny_case(2, B=2, Hq=4, Hkv=2, Tq=2, Tmax=6, D=8)
    kv_len = np.array([6, 4])
    scale = 0.35
    for causal in (False, True):
        out = A.attention(q, qs, k, ks, v, vs, kv_len, scale, causal=causal)
        for b in range(2):
            L = int(kv_len[b])
            for hq in range(4):
                hkv = hq // 2
                for i in range(2):
                    pos = L - 2 + i
                    ts = [t for t in range(L) if (not causal or t <= pos)]
                    lg = [sum(int(a) * int(c) for a, c in zip(q[b, hq, i], k[b, hkv, t]))
                          * float(qs[b, hq, i]) * float(ks[b, hkv, t]) * scale for t in ts]
                    mx = max(lg)
                    w = [math.exp(x - mx) for x in lg]
                    tot = sum(w)
                    for d in range(8):
                        want = sum(w[j] / tot * int(v[b, hkv, t, d]) * float(vs[b, hkv, t]) for j, t in enumerate(ts))
                        assert abs(out[b, hq, i, d] - want) <= 1e-12 * max(1.0, abs(want))


def test_uniform_softmax_gives_mean_and_single_token_gives_value():
    q, qs, k, ks, v, vs = _tiny_case(3)
    k[:] = k[:, :, :1, :]                              # identical keys -> equal logits
    ks[:] = ks[:, :, :1]
    out = A.attention(q, qs, k, ks, v, vs, np.array([6]), 0.1)
    deq = Q.dequantize(v, vs)
    for hq in range(4):
        np.testing.assert_allclose(out[0, hq, 0], deq[0, hq // 2].mean(axis=0), rtol=1e-13, atol=1e-15)
    out1 = A.attention(q, qs, k, ks, v, vs, np.array([1]), 0.1)
    for hq in range(4):
        np.testing.assert_allclose(out1[0, hq, 0], deq[0, hq // 2, 0], rtol=1e-15)


def test_one_hot_logit_and_gqa_head_mapping():
    q, qs, k, ks, v, vs = _tiny_case(4, Hq=4, Hkv=2)
    q[:] = 0; q[..., 0] = 1000
    k[:] = 0; k[:, :, 3, 0] = 1000                     # token 3 dominates every head
    qs[:] = 1e-2; ks[:] = 1e-2
    out = A.attention(q, qs, k, ks, v, vs, np.array([6]), 1.0)
    deq = Q.dequantize(v, vs)
    for hq in range(4):
        np.testing.assert_allclose(out[0, hq, 0], deq[0, hq // 2, 3], rtol=1e-12)
    assert not np.allclose(out[0, 0, 0], out[0, 2, 0])  # heads 0-1 read KV head 0, heads 2-3 read KV head 1


def test_causal_first_query_sees_only_first_token():
    q, qs, k, ks, v, vs = _tiny_case(5, Tq=6, Tmax=6)
    out = A.attention(q, qs, k, ks, v, vs, np.array([6]), 0.2, causal=True)
    deq = Q.dequantize(v, vs)
    for hq in range(4):
        np.testing.assert_allclose(out[0, hq, 0], deq[0, hq // 2, 0], rtol=1e-15)


def test_queries_before_the_first_token_give_zero_rows():
    # causal, kv_len 3 < Tq 6: queries 0..2 sit at positions -3..-1 and see nothing (O = 0);
    # queries 3..5 are the queries at positions 0..2 of a 3-token context
    q, qs, k, ks, v, vs = _tiny_case(7, Tq=6, Tmax=6)
    out = A.attention(q, qs, k, ks, v, vs, np.array([3]), 0.2, causal=True)
    assert np.all(out[:, :, :3] == 0.0)
    ref = A.attention(q[:, :, 3:], qs[:, :, 3:], k, ks, v, vs, np.array([3]), 0.2, causal=True)
    np.testing.assert_array_equal(out[:, :, 3:], ref)
    deq = Q.dequantize(v, vs)
    for hq in range(4):   # the first of them sees only token 0
        np.testing.assert_allclose(out[0, hq, 3], deq[0, hq // 2, 0], rtol=1e-15)
