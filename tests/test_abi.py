"""The C ABI: the library loads without a GPU and exports every symbol include/heal.h
declares; host-side validation rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import error_compensated_gemm_b200 as heal

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "heal.h")).read()
    return sorted(set(re.findall(r"^\s*(?:heal_status_t|size_t|const char\*)\s+(heal_\w+)\s*\(", src, re.M)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(heal.EXPORTED)


def test_library_loads_and_exports_every_symbol():
    L = heal.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert heal.heal_version().startswith("heal-b200")
    assert heal.status_string(heal.HEAL_ERR_TIMEOUT) == "a device-side wait ran out of time"


def test_workspace_queries_are_host_only():
    # chunk values [64][1][4096] FP32
    assert heal.heal_gemm_workspace_bytes(1, 4096, 4096, heal.TILE_SKINNY_SPLITK) == 64 * 4096 * 4
    assert heal.heal_gemm_workspace_bytes(4096, 4096, 4096, heal.TILE_128x128) == 0
    # a split pass over B adds its hi and lo parts (2 + 2 bytes per element) after the split-K part
    assert heal.heal_gemm_workspace_bytes(4096, 14336, 4096, b_split_pass=True) == 4 * 4096 * 14336
    assert heal.heal_gemm_workspace_bytes(1, 4096, 4096, heal.TILE_SKINNY_SPLITK, b_split_pass=True) == \
        64 * 4096 * 4 + 4 * 4096 * 4096
    assert heal.heal_attention_workspace_bytes(8, 32, 1, 8192) > 0
    assert heal.heal_attention_workspace_bytes(0, 32, 1, 8192) == 0
    # decode shapes ((Hq/Hkv)*Tq <= 8) need the split-context partials only; prefill shapes
    # the byte planes: 6 B per cache element + 2 B per query element + s_v*2^E + E
    dec = heal.heal_attention_workspace_bytes_gqa(8, 32, 8, 2, 8192)
    assert 0 < dec <= heal.heal_attention_workspace_bytes(8, 32, 2, 8192)
    assert heal.heal_attention_workspace_bytes_gqa(1, 32, 8, 512, 640) == \
        6 * 8 * 640 * 128 + 2 * 32 * 512 * 128 + 4 * 8 * 640 + 128
    # the short form is an upper bound for every Hkv dividing Hq
    for hkv in (1, 2, 4, 8, 16, 32):
        assert heal.heal_attention_workspace_bytes_gqa(2, 32, hkv, 96, 192) <= heal.heal_attention_workspace_bytes(2, 32, 96, 192)
    assert heal.heal_attention_workspace_bytes_gqa(1, 30, 8, 4, 64) == 0   # Hq % Hkv != 0


def test_invalid_arguments_rejected_before_launch():
    L = heal.lib()
    o = heal.gemm_opts()
    # null pointers / bad sizes: rejected on the host, no CUDA call needed
    assert L.heal_gemm_compensated(0, 4, 4, None, 4, None, 4, None, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    assert L.heal_gemm_compensated(4, 4, 4, None, 4, None, 4, None, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    assert L.heal_gemm_compensated(4, 4, 4, fake, 3, fake, 4, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 4, fake, 4, 7, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.reserved[0] = 1
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 4, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.reserved[0] = 0
    o.b_static = 2                                   # only 0 / 1
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 8, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.b_static = 0
    o.b_presplit = 3                                 # only 0 / 1 / 2
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 8, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.b_presplit = 1                                 # pre-split B needs its lo part
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 8, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.b_presplit = 2                                 # a 16-bit B has no lo part
    o.b_lo = 1 << 20
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 8, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.b_lo = None
    assert L.heal_gemm_compensated(4, 4, 4, fake, 4, fake, 4, fake, 4, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT  # ldb % 8
    o.b_presplit = 0
    o.b_split_pass = 2                               # only 0 / 1
    assert L.heal_gemm_compensated(4, 8, 8, fake, 8, fake, 8, fake, 8, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.b_split_pass = 1                               # no workspace for B's parts
    assert L.heal_gemm_compensated(4, 8, 8, fake, 8, fake, 8, fake, 8, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    o.workspace, o.workspace_bytes = 1 << 20, 4 * 8 * 8
    assert L.heal_gemm_compensated(4, 8, 8, fake, 8, fake, 16, fake, 8, 0, ctypes.byref(o), None) == heal.HEAL_ERR_UNSUPPORTED  # B not contiguous
    o.b_presplit, o.b_lo = 1, 1 << 20                # a split pass over a pre-split B makes no sense
    assert L.heal_gemm_compensated(4, 8, 8, fake, 8, fake, 8, fake, 8, 0, ctypes.byref(o), None) == heal.HEAL_ERR_INVALID_ARGUMENT
    with pytest.raises(ValueError):
        heal.gemm_opts(b_lo=object(), b_16bit=True)
    assert L.heal_split(fake, fake, fake, -1, 0, None) == heal.HEAL_ERR_INVALID_ARGUMENT
    assert L.heal_split(None, None, None, 0, 0, None) == heal.HEAL_OK       # n == 0 is a no-op
    assert L.heal_kv_quantize_int16(fake, 1, 1, 1, 1, 96, 96, 96, 96, fake, fake, 1, 0, None) == heal.HEAL_ERR_UNSUPPORTED
    assert L.heal_kv_quantize_int16(fake, 1, 1, 2, 1, 128, 256, 128, 128, fake, fake, 1, 0, None) == heal.HEAL_ERR_INVALID_ARGUMENT
    assert L.heal_attention_int16(fake, fake, fake, fake, fake, fake, 1, 32, 8, 256, 1, fake, 64, 0.1, 0, fake,
                                  fake, 1 << 20, None, None) == heal.HEAL_ERR_UNSUPPORTED
    assert L.heal_attention_int16(fake, fake, fake, fake, fake, fake, 1, 30, 8, 128, 1, fake, 64, 0.1, 0, fake,
                                  fake, 1 << 20, None, None) == heal.HEAL_ERR_INVALID_ARGUMENT


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(8)
    with pytest.raises(ValueError):
        heal.heal_split(x, torch.zeros(8, dtype=torch.int16), torch.zeros(8, dtype=torch.int16))
