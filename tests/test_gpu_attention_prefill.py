"""GPU parity of the prefill attention kernel (heal_attention_int16 with more than 8 query
rows per KV head: 128-row query tiles on the tcgen05 tensor cores) against the oracle,
through the C ABI.

Inputs are quantized on the CPU by the oracle (oracle.quant) from the seeded bf16 workload;
no expected value comes from the CUDA path.
  * S_int (exact integer QK^T through the test hook) must be bit-identical to int64 dots.
  * O is compared with the FP64 definition under the decode tests' bound,
        ||O - O_ref|| / ||O_ref||  <=  4 * (x_max + 8) * 2^-23 + 1e-6.
    The prefill kernel forms logit * log2(e) from fp32(S_int) with two FP32 products
    (relative error <= 3 * 2^-24 of |x|), evaluates 2^x with the hardware approximation
    (relative error about 2^-22) against a reference maximum that may trail the row maximum
    by up to 8 (P <= 2^8, the same relative precision), and
    adds each 64-token block's tensor-core PV product into FP32 with round-to-nearest, so
    each weight carries about (1.5 |x| + 10) * 2^-23 of relative error: inside the bound.
"""
import math

import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
from oracle import attention as OA
from tests.gpu_helpers import dev, status_ok, to_np
from tests.test_gpu_attention import assert_rows_within, check, make_inputs, run_gpu, tolerance

pytestmark = pytest.mark.gpu

SCALE = 128 ** -0.5


def test_prefill_causal_ragged_tiles():
    # 200 queries = one full and one ragged 128-row tile; 4 key blocks, the last ragged
    q, qs, kq, kss, vq, vss = make_inputs(B=1, Hq=4, Hkv=1, D=128, T=200, Tq=200, Tmax=256)
    check(q, qs, kq, kss, vq, vss, [200], SCALE, causal=True)


def test_prefill_gqa_noncausal_two_batches():
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=8, Hkv=2, D=128, T=300, Tq=130, Tmax=320)
    check(q, qs, kq, kss, vq, vss, [300, 150], SCALE, causal=False)


def test_prefill_chunked_causal_queries_at_the_end():
    # 150 queries at positions 250..399 of a 400-token context
    q, qs, kq, kss, vq, vss = make_inputs(B=1, Hq=8, Hkv=2, D=128, T=400, Tq=150, Tmax=448)
    check(q, qs, kq, kss, vq, vss, [400], SCALE, causal=True)


def test_prefill_few_rows_per_kv_head_group():
    # (Hq/Hkv) * Tq = 4 * 3 = 12 > 8: a short multi-token step also takes the tcgen05 path
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=8, Hkv=2, D=128, T=256, Tq=3, Tmax=256)
    check(q, qs, kq, kss, vq, vss, [256, 70], SCALE, causal=True)


def test_prefill_context_shorter_than_queries_gives_zero_rows():
    # causal, kv_len 60 < Tq 100: queries 0..39 sit before the first token and see nothing
    q, qs, kq, kss, vq, vss = make_inputs(B=1, Hq=4, Hkv=4, D=128, T=100, Tq=100, Tmax=128)
    out, qk = run_gpu(q, qs, kq, kss, vq, vss, [60], SCALE, causal=True, hook=True)
    assert np.all(out[:, :, :40] == 0.0)
    # the others are the queries at positions 0..59 of a 60-token context
    q2, qs2 = q[:, :, 40:], qs[:, :, 40:]
    ref, s_blocks = OA.attention(q2, qs2, kq, kss, vq, vss, [60], SCALE, causal=True, return_s_int=True)
    for i in range(60):
        np.testing.assert_array_equal(qk[0, :, 40 + i, :i + 1], s_blocks[0][:, i, :i + 1])
    tol = tolerance(q2, qs2, kq, kss, [60], SCALE, 4)
    err = np.linalg.norm(out[:, :, 40:] - ref) / np.linalg.norm(ref)
    assert err <= tol, (err, tol)


def test_prefill_bitwise_repeatable():
    q, qs, kq, kss, vq, vss = make_inputs(B=1, Hq=8, Hkv=2, D=128, T=640, Tq=640, Tmax=640, seed=3)
    a, _ = run_gpu(q, qs, kq, kss, vq, vss, [640], SCALE, causal=True)
    b, _ = run_gpu(q, qs, kq, kss, vq, vss, [640], SCALE, causal=True)
    assert np.array_equal(a, b)


def test_prefill_extreme_int16_values_exact_dots():
    B, Hq, Hkv, D, T, Tq = 1, 2, 1, 128, 192, 16
    rng = np.random.default_rng(7)
    q = np.full((B, Hq, Tq, D), -32767, np.int16)
    q[0, 1] = 32767
    q[0, 0, 3, ::2] = -32768
    q[0, 1, 5] = rng.integers(-32768, 32768, D).astype(np.int16)
    kq = np.full((B, Hkv, T, D), 32767, np.int16)
    kq[0, 0, 5] = -32767
    kq[0, 0, 6, ::3] = 255
    kq[0, 0, 100:] = rng.integers(-32768, 32768, (T - 100, D)).astype(np.int16)
    vq = rng.integers(-32767, 32768, (B, Hkv, T, D)).astype(np.int16)
    qs = np.full((B, Hq, Tq), 1e-9, np.float32)
    kss = np.full((B, Hkv, T), 1e-9, np.float32)
    vss = rng.uniform(1e-6, 1e-3, (B, Hkv, T)).astype(np.float32)
    check(q, qs, kq, kss, vq, vss, [T], 0.5, causal=True)


def test_prefill_extreme_v_scales():
    # V scales near the FP32 extremes: the per-(batch, kv head) power of two must stay exact
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=4, Hkv=2, D=128, T=256, Tq=130, Tmax=256, seed=5)
    vss = vss.copy()
    vss[0] *= np.float32(1e30)
    vss[1] *= np.float32(1e-30)
    check(q, qs, kq, kss, vq, vss, [256, 256], SCALE, causal=True)


def test_prefill_full_size_sampled_rows():
    """Causal self-attention over an 8192-token prompt, 32 query heads on 8 KV heads, in the
    configuration the benchmark times.  1024 query rows are checked against the oracle: for
    every head a block of 32 consecutive positions, the blocks spread from the first
    positions to the last and across 128-row tile edges; each row on its own bound."""
    B, Hq, Hkv, D, T = 1, 32, 8, 128, 8192
    q, qs, kq, kss, vq, vss = make_inputs(B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, Tq=T)
    out, _ = run_gpu(q, qs, kq, kss, vq, vss, [T], SCALE, causal=True)
    assert np.all(np.isfinite(out))
    n = 32
    vabs = np.abs(np.asarray(vq, np.int64))
    checked = 0
    for h in range(Hq):
        p = min(T - 1, n - 1 + (h * (T - n)) // (Hq - 1) + (h % 3) * 37)     # last position of the block
        g = h // (Hq // Hkv)
        sl = (slice(None), slice(h, h + 1), slice(p + 1 - n, p + 1))
        kv = (kq[:, g:g + 1], kss[:, g:g + 1])
        ref = OA.attention(q[sl], qs[sl], *kv, vq[:, g:g + 1], vss[:, g:g + 1], [p + 1], SCALE, causal=True)
        abs_ref = OA.attention(q[sl], qs[sl], *kv, vabs[:, g:g + 1], vss[:, g:g + 1], [p + 1], SCALE, causal=True)
        tol = tolerance(q[sl], qs[sl], kq[:, g:g + 1, :p + 1], kss[:, g:g + 1, :p + 1], [p + 1], SCALE, 1)
        assert_rows_within(out[sl], ref, abs_ref, tol)
        checked += n
    assert checked == 1024


def test_prefill_workspace_sizes():
    exact = heal.heal_attention_workspace_bytes_gqa(1, 32, 8, 8192, 8192)
    assert exact == 6 * 8 * 8192 * 128 + 2 * 32 * 8192 * 128 + 4 * 8 * 8192 + 128
    assert heal.heal_attention_workspace_bytes(1, 32, 8192, 8192) >= exact
    # a workspace one byte short is refused before any launch
    d = dev()
    B, Hq, Hkv, D, Tq, Tmax = 1, 4, 1, 128, 64, 64
    i16 = lambda *s: torch.zeros(s, dtype=torch.int16, device=d)
    f32 = lambda *s: torch.ones(s, dtype=torch.float32, device=d)
    need = heal.heal_attention_workspace_bytes_gqa(B, Hq, Hkv, Tq, Tmax)
    ws = torch.empty(need, dtype=torch.uint8, device=d)
    out = torch.empty(B, Hq, Tq, D, device=d)
    kv_len = torch.full((B,), Tmax, dtype=torch.int32, device=d)
    with pytest.raises(heal.HealError):
        heal.heal_attention_int16(i16(B, Hq, Tq, D), f32(B, Hq, Tq), i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax),
                                  i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax), kv_len, SCALE, out, ws[:need - 16])
    heal.heal_attention_int16(i16(B, Hq, Tq, D), f32(B, Hq, Tq), i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax),
                              i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax), kv_len, SCALE, out, ws)
    status_ok()
    # all-zero Q and K: uniform softmax over zero V gives zeros
    assert torch.all(out == 0)


def test_prefill_head_dim_64_is_unsupported():
    d = dev()
    B, Hq, Hkv, D, Tq, Tmax = 1, 4, 1, 64, 64, 64
    i16 = lambda *s: torch.zeros(s, dtype=torch.int16, device=d)
    f32 = lambda *s: torch.ones(s, dtype=torch.float32, device=d)
    ws = torch.empty(heal.heal_attention_workspace_bytes(B, Hq, Tq, Tmax), dtype=torch.uint8, device=d)
    with pytest.raises(heal.HealError):
        heal.heal_attention_int16(i16(B, Hq, Tq, D), f32(B, Hq, Tq), i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax),
                                  i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax),
                                  torch.full((B,), Tmax, dtype=torch.int32, device=d), 64 ** -0.5,
                                  torch.empty(B, Hq, Tq, D, device=d), ws)


def test_prefill_tiles_with_no_visible_token():
    # causal, kv_len 100 < Tq 300: the first 128-row tile sees no token at all (its CTA
    # loads nothing and writes zeros); rows 0..199 are zero, rows 200..299 are the queries
    # at positions 0..99
    q, qs, kq, kss, vq, vss = make_inputs(B=1, Hq=4, Hkv=2, D=128, T=300, Tq=300, Tmax=320, seed=9)
    out, _ = run_gpu(q, qs, kq, kss, vq, vss, [100], SCALE, causal=True)
    ref = OA.attention(q, qs, kq, kss, vq, vss, [100], SCALE, causal=True)
    assert np.all(out[:, :, :200] == 0.0)
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert err <= tolerance(q[:, :, 200:], qs[:, :, 200:], kq, kss, [100], SCALE, 2), err
