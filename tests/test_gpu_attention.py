"""GPU parity of heal_attention_int16 against the oracle, through the C ABI.

Inputs are quantized on the CPU by the oracle (oracle.quant) from the seeded bf16
workload, so no expected value comes from the CUDA path.
  * S_int (exact integer QK^T, via the test hook) must be bit-identical to int64 dots.
  * O is compared with the FP64 definition.  Tolerance: the device rounds each logit to
    FP32 (relative 2^-24), scales by log2(e) in FP32 and evaluates exp2 in FP32, so each
    weight carries a relative error of about (|x| + 8) * 2^-23 where |x| is the largest
    |logit * log2 e| in play; P is carried in two FP16 parts (2^-22) and the products are
    accumulated in FP32.  The test bound is
        ||O - O_ref|| / ||O_ref||  <=  4 * (x_max + 8) * 2^-23 + 1e-6
    which is about 1e-5 at x_max ~ 12 and grows only with extreme logits.
    The same bound holds row by row once it is taken relative to the softmax-weighted sum
    of |v| (each weight's error multiplies |v_t|, never v_t's signed sum), so every query
    row is also checked on its own:
        ||O_row - O_ref_row|| <= tol * || sum_t p_t |v_t| ||_row
    which localises one bad head or query that the whole-tensor ratio would average away.
"""
import math

import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
import synthetic
from oracle import attention as OA
from oracle import quant as Q
from tests.gpu_helpers import dev, status_ok, to_np

pytestmark = pytest.mark.gpu


def make_inputs(B, Hq, Hkv, D, T, Tq=1, Tmax=None, seed=0):
    Tmax = Tmax or T
    Qb, K, V = synthetic.kv_decode(B=B, T=T, Hkv=Hkv, Hq=Hq, D=D, Tq=Tq, seeds=(2 + seed, 3 + seed, 4 + seed))
    q, qs = Q.quantize_kv(Qb.float().numpy())            # [B, Hq, Tq, D]
    kq, kss = Q.quantize_kv(K.float().numpy())           # [B, Hkv, T, D]
    vq, vss = Q.quantize_kv(V.float().numpy())
    if Tmax > T:                                         # cache rows beyond T: arbitrary junk
        rng = np.random.default_rng(99)
        pad = lambda a, fill: np.concatenate([a, fill(a.shape[:2] + (Tmax - T,) + a.shape[3:])], axis=2)
        kq = pad(kq, lambda s: rng.integers(-32767, 32768, s).astype(np.int16))
        vq = pad(vq, lambda s: rng.integers(-32767, 32768, s).astype(np.int16))
        kss = pad(kss, lambda s: np.full(s, np.nan, np.float32))
        vss = pad(vss, lambda s: np.full(s, np.inf, np.float32))
    return q, qs, kq, kss, vq, vss


def run_gpu(q, qs, kq, kss, vq, vss, kv_len, scale, causal=False, hook=False):
    d = dev()
    B, Hq, Tq, D = q.shape
    Tmax = kq.shape[2]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(d)
    out = torch.full((B, Hq, Tq, D), float("nan"), device=d)
    ws = torch.empty(heal.heal_attention_workspace_bytes(B, Hq, Tq, Tmax) // 4, dtype=torch.float32, device=d)
    qk = torch.full((B, Hq, Tq, Tmax), -(2 ** 62), dtype=torch.int64, device=d) if hook else None
    heal.heal_attention_int16(t(q), t(qs), t(kq), t(kss), t(vq), t(vss), t(np.asarray(kv_len, np.int32)), scale,
                              out, ws, causal=causal, qk_int_out=qk)
    status_ok()
    return to_np(out).astype(np.float64), (to_np(qk) if hook else None)


def tolerance(q, qs, kq, kss, kv_len, scale, Hkv):
    x_max = 0.0
    G = q.shape[1] // Hkv
    for b in range(q.shape[0]):
        L = int(kv_len[b])
        for h in range(q.shape[1]):
            S = OA.qk_int(q[b, h], kq[b, h // G, :L]).astype(np.float64)
            lg = S * qs[b, h][:, None].astype(np.float64) * kss[b, h // G, :L].astype(np.float64) * scale
            x_max = max(x_max, float(np.max(np.abs(lg))) * math.log2(math.e))
    return 4 * (x_max + 8) * 2.0 ** -23 + 1e-6


def check(q, qs, kq, kss, vq, vss, kv_len, scale, causal=False, hook=True):
    out, qk = run_gpu(q, qs, kq, kss, vq, vss, kv_len, scale, causal=causal, hook=hook)
    ref, s_blocks = OA.attention(q, qs, kq, kss, vq, vss, kv_len, scale, causal=causal, return_s_int=True)
    if hook:
        B, Hq, Tq, _ = q.shape
        for b in range(B):
            L = int(kv_len[b])
            for i in range(Tq):
                vis = np.arange(L) <= (L - Tq + i) if causal else np.ones(L, bool)
                np.testing.assert_array_equal(qk[b, :, i, :L][:, vis], s_blocks[b][:, i, :][:, vis])
    tol = tolerance(q, qs, kq, kss, kv_len, scale, kq.shape[1])
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert np.all(np.isfinite(out))
    assert err <= tol, (err, tol)
    abs_ref = OA.attention(q, qs, kq, kss, np.abs(np.asarray(vq, np.int64)), vss, kv_len, scale, causal=causal)
    assert_rows_within(out, ref, abs_ref, tol)
    return err


def assert_rows_within(out, ref, abs_ref, tol):
    """Per query row: ||out - ref|| <= tol * ||sum_t p_t |v_t||| (rows that see no token
    must be exactly zero on both sides)."""
    d = np.linalg.norm((out - ref).reshape(-1, out.shape[-1]), axis=1)
    a = np.linalg.norm(abs_ref.reshape(-1, out.shape[-1]), axis=1)
    bad = np.nonzero(d > tol * a)[0]
    assert bad.size == 0, [(int(r), float(d[r]), float(tol * a[r])) for r in bad[:8]]


def test_decode_gqa_ragged_lengths():
    q, qs, kq, kss, vq, vss = make_inputs(B=3, Hq=8, Hkv=2, D=128, T=256, Tmax=384)
    check(q, qs, kq, kss, vq, vss, [256, 100, 1], 128 ** -0.5)


def test_decode_head_dim_64():
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=8, Hkv=4, D=64, T=320)
    check(q, qs, kq, kss, vq, vss, [320, 77], 64 ** -0.5)


def test_multi_query_causal():
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=8, Hkv=4, D=128, T=192, Tq=4)
    check(q, qs, kq, kss, vq, vss, [192, 130], 128 ** -0.5, causal=True)


@pytest.mark.parametrize("Hq,Hkv,Tq", [(6, 2, 1), (6, 2, 2), (8, 2, 1), (10, 2, 1)])
def test_decode_row_counts_packed_and_unpacked(Hq, Hkv, Tq):
    """R = (Hq/Hkv)*Tq query rows per KV head: 3 and 4 take the form whose PV fragments carry
    P_hi in columns 0-3 and the residual in columns 4-7; 6 takes the four-product form; 5
    rows run through the same form."""
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=Hq, Hkv=Hkv, D=128, T=320, Tq=Tq)
    check(q, qs, kq, kss, vq, vss, [320, 199], 128 ** -0.5, causal=Tq > 1)


def test_mha_and_many_blocks():
    q, qs, kq, kss, vq, vss = make_inputs(B=1, Hq=4, Hkv=4, D=128, T=4096)
    check(q, qs, kq, kss, vq, vss, [4001], 128 ** -0.5)


def test_extreme_int16_values_exact_dots():
    B, Hq, Hkv, D, T = 1, 4, 1, 128, 128
    q = np.full((B, Hq, 1, D), -32767, np.int16)
    q[0, 1] = 32767
    q[0, 2, 0, ::2] = -32768
    kq = np.full((B, Hkv, T, D), 32767, np.int16)
    kq[0, 0, 5] = -32767
    kq[0, 0, 6, ::3] = 255
    vq = np.random.default_rng(1).integers(-32767, 32768, (B, Hkv, T, D)).astype(np.int16)
    qs = np.full((B, Hq, 1), 1e-9, np.float32)
    kss = np.full((B, Hkv, T), 1e-9, np.float32)
    vss = np.full((B, Hkv, T), 1e-4, np.float32)
    check(q, qs, kq, kss, vq, vss, [T], 0.5)


def test_extreme_v_scales():
    """V scales from 3e-38 up to 3e33: the per-block power of two 2^E that brings the largest
    V scale into [32, 64) then lies outside FP32's normal range on both ends; the kernel applies
    it in two exact steps.  Blocks of tiny and huge scales alternate, so E also moves down."""
    B, Hq, Hkv, D, T = 1, 4, 1, 128, 320
    q, qs, kq, kss, vq, vss = make_inputs(B=B, Hq=Hq, Hkv=Hkv, D=D, T=T)
    vss = vss.copy()
    vss[0, 0, :128] *= np.float32(3e-38 / float(vss[0, 0, :128].max()))   # first two blocks: tiny
    vss[0, 0, 192:256] *= np.float32(3e33 / float(vss[0, 0, 192:256].max()))   # fourth block: huge
    assert np.all(np.isfinite(vss))
    check(q, qs, kq, kss, vq, vss, [T], D ** -0.5)


def test_repeat_runs_bitwise_identical():
    q, qs, kq, kss, vq, vss = make_inputs(B=2, Hq=8, Hkv=2, D=128, T=1024)
    a, _ = run_gpu(q, qs, kq, kss, vq, vss, [1024, 900], 128 ** -0.5)
    for _ in range(3):
        b, _ = run_gpu(q, qs, kq, kss, vq, vss, [1024, 900], 128 ** -0.5)
        assert np.array_equal(a, b)


def test_full_size_decode_config():
    """B=8, Hq=32, Hkv=8, D=128, context 8192, one query token: exact S_int on every
    (head, token) and O against the FP64 definition."""
    q, qs, kq, kss, vq, vss = make_inputs(B=8, Hq=32, Hkv=8, D=128, T=8192)
    err = check(q, qs, kq, kss, vq, vss, [8192] * 8, 128 ** -0.5)
    print("full-size normwise error", err)
