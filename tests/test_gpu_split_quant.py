"""GPU parity of heal_split (bit-exact hi/lo encodings) and heal_kv_quantize_int16
(bit-exact INT16 codes and FP32 scales) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
import synthetic
from oracle import quant as Q
from oracle import split as S
from tests.gpu_helpers import dev, status_ok, to_np

pytestmark = pytest.mark.gpu


def special_values():
    return np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 2.0 ** -24, 2.0 ** -25, 1.0 + 2.0 ** -11,
                     1.0 + 3 * 2.0 ** -11, 3.0e-5, -7.0e-8, 1e-30, 12345.678, 0.1, 1e30], np.float32)


@pytest.mark.parametrize("fmt,name", [(heal.SPLIT_FP16_S11, S.FP16_S11), (heal.SPLIT_BF16, S.BF16)])
@pytest.mark.parametrize("n,offset", [(1 << 20, 0), (1000003, 0), (4099, 1), (7, 0), (0, 0)])
def test_split_bit_exact(fmt, name, n, offset):
    d = dev()
    x = synthetic.normal((n,), seed=n % 97, std=3.0).numpy()
    x[: min(n, 16)] = special_values()[: min(n, 16)]
    if name == S.FP16_S11:
        x = np.where(np.abs(x) > 6e4, 1.0, x).astype(np.float32)   # keep FP16 hi finite
    buf = torch.zeros(n + offset, dtype=torch.float32, device=d)
    xd = buf[offset:]
    xd.copy_(torch.from_numpy(x))
    hi = torch.empty(n, dtype=torch.int16, device=d)
    lo = torch.empty(n, dtype=torch.int16, device=d)
    heal.heal_split(xd, hi, lo, fmt)
    status_ok()
    _, _, hb, lb = S.split(x, name)
    np.testing.assert_array_equal(to_np(hi).view(np.uint16), hb)
    np.testing.assert_array_equal(to_np(lo).view(np.uint16), lb)


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("D", [128, 64])
def test_kv_quantize_bit_exact(in_dtype, D):
    d = dev()
    B, T, H, Tmax, t_off = 2, 300, 8, 512, 17
    _, K, _ = synthetic.kv_decode(B=B, T=T, Hkv=H, Hq=32, D=D)
    x = K.to(in_dtype)
    x[0, 3, 2] = 0                                  # an all-zero row
    x[1, 5, 1] = 0.375                              # a constant row
    xd = x.to(d)
    qc = torch.full((B, H, Tmax, D), 7, dtype=torch.int16, device=d)
    sc = torch.full((B, H, Tmax), -1.0, dtype=torch.float32, device=d)
    heal.heal_kv_quantize_int16(xd, qc, sc, t_offset=t_off)
    status_ok()
    q_ref, s_ref = Q.quantize_kv(x.float().numpy())
    qn, sn = to_np(qc), to_np(sc)
    np.testing.assert_array_equal(qn[:, :, t_off:t_off + T], q_ref)
    np.testing.assert_array_equal(sn[:, :, t_off:t_off + T].view(np.uint32), s_ref.view(np.uint32))
    assert np.all(qn[:, :, :t_off] == 7) and np.all(qn[:, :, t_off + T:] == 7)   # other rows untouched
    assert np.all(sn[:, :, :t_off] == -1.0) and np.all(sn[:, :, t_off + T:] == -1.0)


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("D,H", [(8, 3), (16, 5), (32, 12), (128, 12), (128, 40), (256, 5)])
def test_kv_quantize_head_dims_and_ragged_head_groups(in_dtype, D, H):
    """Every row-group width (8 lanes' worth of values per lane group: D = 8 .. 256) and
    head counts that leave the last group of a token partly empty; one row of half-integer
    products (absmax 65534 -> inv = 0.5 exactly, odd inputs) checks that ties round to
    even."""
    d = dev()
    B, T, Tmax, t_off = 2, 67, 80, 5
    g = torch.Generator().manual_seed(1000 + D + H)
    x = (torch.randn(B, T, H, D, generator=g) * torch.exp(torch.randn(B, T, H, 1, generator=g))).to(in_dtype)
    x[1, 2, H - 1] = 0
    if in_dtype == torch.float32:
        row = torch.arange(D, dtype=torch.float32) * 2 - (D - 1)     # odd values
        row[0] = 65534.0
        x[0, 1, 0] = row
    qc = torch.full((B, H, Tmax, D), 7, dtype=torch.int16, device=d)
    sc = torch.full((B, H, Tmax), -1.0, dtype=torch.float32, device=d)
    heal.heal_kv_quantize_int16(x.to(d), qc, sc, t_offset=t_off)
    status_ok()
    q_ref, s_ref = Q.quantize_kv(x.float().numpy())
    qn, sn = to_np(qc), to_np(sc)
    np.testing.assert_array_equal(qn[:, :, t_off:t_off + T], q_ref)
    np.testing.assert_array_equal(sn[:, :, t_off:t_off + T].view(np.uint32), s_ref.view(np.uint32))
    assert np.all(qn[:, :, :t_off] == 7) and np.all(qn[:, :, t_off + T:] == 7)
    assert np.all(sn[:, :, :t_off] == -1.0) and np.all(sn[:, :, t_off + T:] == -1.0)
    if in_dtype == torch.float32:
        # 0.5 * odd k is a tie; the even neighbour wins
        k = np.arange(D) * 2 - (D - 1)
        want = np.rint(k[1:] * 0.5).astype(np.int16)
        assert np.array_equal(qn[0, 0, t_off + 1, 1:], want) and qn[0, 0, t_off + 1, 0] == 32767


def test_kv_quantize_strided_input_and_full_size():
    """Config-sized K cache (B=8, T=8192, Hkv=8, D=128) from a strided view: bit-exact on
    every row."""
    d = dev()
    _, K, _ = synthetic.kv_decode()
    big = torch.zeros(8, 8192, 8, 136, dtype=torch.bfloat16)
    big[..., :128] = K
    xd = big.to(d)[..., :128]                        # head stride 136: not contiguous
    qc = torch.empty(8, 8, 8192, 128, dtype=torch.int16, device=d)
    sc = torch.empty(8, 8, 8192, dtype=torch.float32, device=d)
    heal.heal_kv_quantize_int16(xd, qc, sc)
    status_ok()
    q_ref, s_ref = Q.quantize_kv(K.float().numpy())
    np.testing.assert_array_equal(to_np(qc), q_ref)
    np.testing.assert_array_equal(to_np(sc).view(np.uint32), s_ref.view(np.uint32))
