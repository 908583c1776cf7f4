"""Pins for oracle.quant (CPU only).

gist.science technical summary, section 2.A: Q/K/V stored as INT16.  Read as a
symmetric per-(token, head) absmax code in [-32767, 32767], decisions in FP32.
"""
import numpy as np

import synthetic
from oracle import quant as Q


def test_hand_worked_row_with_unit_absmax():
    # absmax = 1 -> inv = 32767 exactly; every product below is exact in FP32
    x = np.array([1.0, -1.0, 0.5, 0.25, 0.0, 2.0 ** -16, 3 * 2.0 ** -16, -0.75], np.float32)
    q, s = Q.quantize_rows(x[None, :])
    # 32767/2 = 16383.5 -> tie -> even 16384; 32767/4 = 8191.75 -> 8192;
    # 32767 * 2**-16 = 0.49998... -> 0; 3 * that = 1.49995... -> 1; -0.75 * 32767 = -24575.25 -> -24575
    np.testing.assert_array_equal(q[0], [32767, -32767, 16384, 8192, 0, 0, 1, -24575])
    assert s[0] == np.float32(1.0) / np.float32(32767.0)


def test_power_of_two_absmax_tie_breaking():
    x = np.array([4.0, 2.0, -1.0, 3.0], np.float32)     # absmax 4: inv = fp32(8191.75) exact
    q, s = Q.quantize_rows(x[None, :])
    # 2 * 8191.75 = 16383.5 -> 16384 (even); -8191.75 -> -8192; 3 * 8191.75 = 24575.25 -> 24575
    np.testing.assert_array_equal(q[0], [32767, 16384, -8192, 24575])
    assert s[0] == np.float32(4.0 / 32767.0)


def test_zero_and_constant_rows():
    x = np.zeros((3, 128), np.float32)
    x[1] = 0.3
    x[2] = -7.25
    q, s = Q.quantize_rows(x)
    assert s[0] == 0 and np.all(q[0] == 0)
    assert np.all(q[1] == 32767) and s[1] == np.float32(np.float32(0.3) / np.float32(32767))
    assert np.all(q[2] == -32767)


def test_roundtrip_bound_and_extremes_on_workload_rows():
    Qb, K, V = synthetic.kv_decode(B=1, T=256, Hkv=8, Hq=32, D=128)
    for t in (Qb, K, V):
        x = t.float().numpy().reshape(-1, 128)
        q, s = Q.quantize_rows(x)
        absmax = np.max(np.abs(x), axis=1)
        err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s[:, None].astype(np.float64))
        bound = s[:, None].astype(np.float64) / 2 + 2.0 ** -22 * absmax[:, None]
        assert np.all(err <= bound)
        assert np.all(np.max(np.abs(q.astype(np.int32)), axis=1) == 32767)
        assert q.min() >= -32767
        # the element at absmax maps to +-32767 with its own sign
        idx = np.argmax(np.abs(x), axis=1)
        rows = np.arange(x.shape[0])
        np.testing.assert_array_equal(np.sign(x[rows, idx]) * 32767, q[rows, idx])


def test_cache_layout_transpose():
    x = synthetic.normal((2, 5, 3, 16), seed=9).numpy()
    qc, sc = Q.quantize_kv(x)
    assert qc.shape == (2, 3, 5, 16) and sc.shape == (2, 3, 5)
    q, s = Q.quantize_rows(x[1, 4, 2][None, :])
    np.testing.assert_array_equal(qc[1, 2, 4], q[0])
    assert sc[1, 2, 4] == s[0]
