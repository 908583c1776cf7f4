"""Helpers shared by the GPU parity tests."""
import numpy as np
import torch

import error_compensated_gemm_b200 as heal


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    heal.lib()   # fail loudly when the extension is missing
    return torch.device("cuda:0")


def status_ok():
    torch.cuda.synchronize()
    st = heal.heal_get_device_status()
    assert st == heal.HEAL_OK, heal.status_string(st)


def to_np(t):
    return t.detach().cpu().numpy()


def padded(t, d):
    """Device copy of a 2-D tensor whose row stride is rounded up to a multiple of 8
    elements (the library needs 16-byte aligned rows)."""
    rows, cols = t.shape
    ld = (cols + 7) // 8 * 8
    store = torch.zeros(rows, ld, dtype=t.dtype, device=d)
    store[:, :cols] = t.to(d)
    return store[:, :cols]


def gemm(A, B, fmt=heal.SPLIT_FP16_S11, tile=heal.TILE_AUTO, b_layout=0, chan_exp=None, b_lo=None, ldc_pad=0):
    """Run heal_gemm_compensated on device copies of numpy/torch inputs; returns numpy C."""
    d = dev()
    A_d = padded(torch.as_tensor(A), d)
    B_d = B if (torch.is_tensor(B) and B.is_cuda) else padded(torch.as_tensor(B), d)
    M, K = A_d.shape
    N = B_d.shape[1] if b_layout == 0 else B_d.shape[0]
    C_full = torch.full((M, N + ldc_pad), float("nan"), device=d)
    C = C_full[:, :N]
    ws = None
    nbytes = heal.heal_gemm_workspace_bytes(M, N, K, tile)
    if nbytes:
        ws = torch.empty(nbytes // 4, dtype=torch.float32, device=d)
    ce = None if chan_exp is None else torch.as_tensor(np.asarray(chan_exp, np.int8)).to(d)
    heal.heal_gemm_compensated(A_d, B_d, C, fmt=fmt, tile_config=tile, chan_exp=ce, b_layout=b_layout,
                               b_lo=b_lo, workspace=ws)
    status_ok()
    return to_np(C).astype(np.float64)
