"""Hand-derived golden fixtures (tests/golden/, derivations and citations in each file).

CPU: the oracle reproduces every fixture.  GPU: the kernels reproduce every fixture
through the C ABI (heal_split, heal_kv_quantize_int16, and the exact integer S of
heal_attention_int16 through its test hook).  Expected values come from the fixture
files only.
"""
import os

import numpy as np
import pytest

from oracle import attention as OA
from oracle import quant as OQ
from oracle import split as OS

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
D_QK = 64


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line


def split_cases(name):
    xs, his, los = [], [], []
    for line in _lines(name):
        x, hi, lo = line.split()
        xs.append(int(x, 16))
        his.append(int(hi, 16))
        los.append(int(lo, 16))
    x = np.array(xs, np.uint32).view(np.float32)
    return x, np.array(his, np.uint16), np.array(los, np.uint16)


def quant_cases():
    rows, codes, scales = [], [], []
    for line in _lines("quant_rows.txt"):
        xs, qs, s = (p.strip() for p in line.split("|"))
        rows.append([float(v) for v in xs.split()])
        codes.append([int(v) for v in qs.split()])
        scales.append(int(s, 16))
    return (np.array(rows, np.float32), np.array(codes, np.int16),
            np.array(scales, np.uint32).view(np.float32))


def pattern(desc, D=D_QK):
    kind, *args = desc.split(":")
    a = [int(v) for v in args]
    v = np.zeros(D, np.int16)
    if kind == "c":
        v[:] = a[0]
    elif kind == "alt":
        v[0::2], v[1::2] = a[0], a[1]
    elif kind == "e0":
        v[0] = a[0]
    elif kind == "ends":
        v[0], v[-1] = a[0], a[1]
    else:
        raise ValueError(desc)
    return v


def qk_cases():
    out = []
    for line in _lines("qk_int_extremes.txt"):
        q, k, s = line.split()
        out.append((q, k, int(s)))
    return out


# ------------------------------------------------------------------ oracle (CPU)
@pytest.mark.parametrize("name,fmt", [("split_fp16_s11.txt", OS.FP16_S11), ("split_bf16.txt", OS.BF16)])
def test_oracle_split_matches_golden(name, fmt):
    x, hi, lo = split_cases(name)
    _, _, hb, lb = OS.split(x, fmt)
    np.testing.assert_array_equal(hb, hi)
    np.testing.assert_array_equal(lb, lo)


def test_oracle_quant_matches_golden():
    x, q, s = quant_cases()
    qo, so = OQ.quantize_rows(x)
    np.testing.assert_array_equal(qo, q)
    np.testing.assert_array_equal(so.view(np.uint32), s.view(np.uint32))


def test_oracle_qk_int_matches_golden():
    for qd, kd, S in qk_cases():
        got = OA.qk_int(pattern(qd)[None, :], pattern(kd)[None, :])
        assert int(got[0, 0]) == S, (qd, kd)


# ------------------------------------------------------------------ kernels (GPU)
@pytest.mark.gpu
@pytest.mark.parametrize("name,fmt", [("split_fp16_s11.txt", 0), ("split_bf16.txt", 1)])
def test_kernel_split_matches_golden(name, fmt):
    import torch

    import error_compensated_gemm_b200 as heal
    from tests.gpu_helpers import dev, status_ok
    d = dev()
    x, hi, lo = split_cases(name)
    xd = torch.from_numpy(x.copy()).to(d)
    h = torch.empty(x.shape, dtype=torch.int16, device=d)
    l = torch.empty_like(h)
    heal.heal_split(xd, h, l, fmt)
    status_ok()
    np.testing.assert_array_equal(h.cpu().numpy().view(np.uint16), hi)
    np.testing.assert_array_equal(l.cpu().numpy().view(np.uint16), lo)


@pytest.mark.gpu
def test_kernel_quant_matches_golden():
    import torch

    import error_compensated_gemm_b200 as heal
    from tests.gpu_helpers import dev, status_ok
    d = dev()
    x, q, s = quant_cases()
    T, D = x.shape
    xd = torch.from_numpy(x.copy()).to(d).view(1, T, 1, D)        # [B, T, H, D]
    qc = torch.full((1, 1, T, D), 12345, dtype=torch.int16, device=d)
    sc = torch.full((1, 1, T), float("nan"), dtype=torch.float32, device=d)
    heal.heal_kv_quantize_int16(xd, qc, sc)
    status_ok()
    np.testing.assert_array_equal(qc[0, 0].cpu().numpy(), q)
    np.testing.assert_array_equal(sc[0, 0].cpu().numpy().view(np.uint32), s.view(np.uint32))


@pytest.mark.gpu
def test_kernel_exact_qk_matches_golden():
    import torch

    import error_compensated_gemm_b200 as heal
    from tests.gpu_helpers import dev, status_ok
    d = dev()
    cases = qk_cases()
    qs = sorted({c[0] for c in cases})
    ks = sorted({c[1] for c in cases})
    Hq, T, Tmax = len(qs), len(ks), 64
    assert Hq <= 8
    q = np.stack([pattern(p) for p in qs])[None, :, None, :]                # [1, Hq, 1, D]
    kc = np.zeros((1, 1, Tmax, D_QK), np.int16)
    kc[0, 0, :T] = np.stack([pattern(p) for p in ks])
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(d)
    scale = np.float32(2.0 ** -16)
    out = torch.empty(1, Hq, 1, D_QK, device=d)
    ws = torch.empty(heal.heal_attention_workspace_bytes(1, Hq, 1, Tmax) // 4, dtype=torch.float32, device=d)
    qk = torch.zeros(1, Hq, 1, Tmax, dtype=torch.int64, device=d)
    heal.heal_attention_int16(t(q), t(np.full((1, Hq, 1), scale, np.float32)), t(kc),
                              t(np.full((1, 1, Tmax), scale, np.float32)), t(np.zeros_like(kc)),
                              t(np.ones((1, 1, Tmax), np.float32)), t(np.array([T], np.int32)), 0.125, out, ws,
                              qk_int_out=qk)
    status_ok()
    S = qk[0, :, 0, :T].cpu().numpy()
    for qd, kd, expect in cases:
        assert int(S[qs.index(qd), ks.index(kd)]) == expect, (qd, kd)
