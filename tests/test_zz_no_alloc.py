"""heal_attention_int16_noalloc: attention for callers that cannot allocate device memory
when they call it (serving loops that allow no allocation after start-up, plugin hosts that
hand an operator only its input and output tensors).  The call keeps its scratch in the
library's fixed device array instead of a caller workspace.

Checked through the C ABI against heal_attention_int16 with a workspace on two calls in a
row with different inputs, so stale scratch from the first call cannot hide in the second.
Both entry points run the same kernels with the same grid, so the results must be the same
bits; the no-alloc result is also held to the oracle's per-row attention bound.  This file
is collected last; it needs nothing from the other tests.
"""
import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
from oracle import attention as OA
from tests.gpu_helpers import dev, status_ok, to_np
from tests.test_gpu_attention import assert_rows_within, make_inputs, tolerance

pytestmark = pytest.mark.gpu

SCALE = 128 ** -0.5


def _dev_inputs(inputs, kv_len, d):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(d)
    q, qs, kq, kss, vq, vss = inputs
    return (t(q), t(qs), t(kq), t(kss), t(vq), t(vss), t(np.asarray(kv_len, np.int32)))


def _run(entry, args, out_shape, d, causal=False):
    B, Hq, Tq, D = out_shape
    out = torch.full(out_shape, float("nan"), device=d)
    if entry == "workspace":
        Tmax = args[2].shape[2]
        ws = torch.empty(heal.heal_attention_workspace_bytes(B, Hq, Tq, Tmax) // 4, device=d)
        heal.heal_attention_int16(*args, SCALE, out, ws, causal=causal)
    else:
        heal.heal_attention_int16_noalloc(*args, SCALE, out, causal=causal)
    status_ok()
    return to_np(out).astype(np.float64)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    d = dev()
    cases = [(make_inputs(B=4, Hq=32, Hkv=8, D=128, T=2048, seed=0), [2048, 1500, 64, 999]),
             (make_inputs(B=2, Hq=32, Hkv=8, D=128, T=1024, seed=7), [1024, 333])]
    for inputs, kv_len in cases:
        args = _dev_inputs(inputs, kv_len, d)
        shape = tuple(inputs[0].shape)
        want = _run("workspace", args, shape, d)
        got = _run("noalloc", args, shape, d)
        assert np.all(np.isfinite(got))
        assert np.array_equal(got, want)
        # and against the oracle, row by row
        q, qs, kq, kss, vq, vss = inputs
        ref = OA.attention(q, qs, kq, kss, vq, vss, kv_len, SCALE)
        abs_ref = OA.attention(q, qs, kq, kss, np.abs(np.asarray(vq, np.int64)), vss, kv_len, SCALE)
        assert_rows_within(got, ref, abs_ref, tolerance(q, qs, kq, kss, kv_len, SCALE, kq.shape[1]))


def test_noalloc_allocates_nothing():
    """After a first call (which looks up the array's address), further calls change neither
    the caching allocator's count nor the device's free memory."""
    d = dev()
    inputs = make_inputs(B=2, Hq=16, Hkv=4, D=128, T=512, seed=3)
    args = _dev_inputs(inputs, [512, 300], d)
    out = torch.empty(tuple(inputs[0].shape), device=d)
    heal.heal_attention_int16_noalloc(*args, SCALE, out)
    status_ok()
    alloc0 = torch.cuda.memory_allocated(d)
    free0, _ = torch.cuda.mem_get_info(d)
    for _ in range(3):
        heal.heal_attention_int16_noalloc(*args, SCALE, out)
    status_ok()
    free1, _ = torch.cuda.mem_get_info(d)
    assert torch.cuda.memory_allocated(d) == alloc0
    assert free1 == free0


def _size_case(B, d):
    Hq = Hkv = 1
    D, Tmax = 128, 64
    rng = np.random.default_rng(B)
    q = rng.integers(-32767, 32768, (B, Hq, 1, D)).astype(np.int16)
    kq = rng.integers(-32767, 32768, (B, Hkv, Tmax, D)).astype(np.int16)
    vq = rng.integers(-32767, 32768, (B, Hkv, Tmax, D)).astype(np.int16)
    qs = np.full((B, Hq, 1), 1e-6, np.float32)
    ks = np.full((B, Hkv, Tmax), 1e-6, np.float32)
    vs = np.full((B, Hkv, Tmax), 1e-4, np.float32)
    kv_len = (1 + np.arange(B) % Tmax).astype(np.int32)
    return _dev_inputs((q, qs, kq, ks, vq, vs), kv_len, d), (B, Hq, 1, D)


def test_noalloc_size_limit_boundary():
    """Decode shapes fit the fixed array up to B * Hq * Tq = 7939: that size runs and gives
    the workspace entry point's bits; 7940 is refused before any launch."""
    d = dev()
    args, shape = _size_case(7939, d)
    want = _run("workspace", args, shape, d)
    got = _run("noalloc", args, shape, d)
    assert np.array_equal(got, want)
    args, shape = _size_case(7940, d)
    out = torch.full(shape, float("nan"), device=d)
    with pytest.raises(heal.HealError) as e:
        heal.heal_attention_int16_noalloc(*args, SCALE, out)
    assert e.value.status == heal.HEAL_ERR_UNSUPPORTED
    assert torch.isnan(out).all()          # nothing was launched


def test_noalloc_prefill_shape_matches_workspace_entry_point():
    # 4 query heads per KV head x 96 queries: the tcgen05 prefill kernel, whose byte planes
    # fit the fixed scratch at this size; the two entry points give the same bits
    d = dev()
    inputs = make_inputs(B=1, Hq=8, Hkv=2, D=128, T=192, Tq=96, seed=11)
    args = _dev_inputs(inputs, [192], d)
    shape = tuple(inputs[0].shape)
    want = _run("workspace", args, shape, d, causal=True)
    got = _run("noalloc", args, shape, d, causal=True)
    assert np.array_equal(got, want)
