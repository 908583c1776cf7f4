"""heal_attention_int16_noalloc: attention for callers that cannot allocate device memory
(stream capture into a CUDA graph, serving loops with a fixed memory budget, plugin hosts
that only hand over input and output tensors).  The call keeps its partial results in the
library's fixed device scratch instead of a caller workspace.

Checked through the C ABI against heal_attention_int16 with a workspace, on two calls in a
row with different inputs, so stale scratch from the first call cannot hide in the second.
This file is collected last; it needs nothing from the other tests.
"""
import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
from tests.gpu_helpers import dev, status_ok, to_np
from tests.test_gpu_attention import make_inputs, tolerance

pytestmark = pytest.mark.gpu


def _run(entry, inputs, kv_len, d):
    q, qs, kq, kss, vq, vss = inputs
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(d)
    B, Hq, Tq, D = q.shape
    out = torch.full((B, Hq, Tq, D), float("nan"), device=d)
    args = (t(q), t(qs), t(kq), t(kss), t(vq), t(vss), t(np.asarray(kv_len, np.int32)), 128 ** -0.5, out)
    if entry == "workspace":
        Tmax = kq.shape[2]
        ws = torch.empty(heal.heal_attention_workspace_bytes(B, Hq, Tq, Tmax) // 4, device=d)
        heal.heal_attention_int16(*args, ws)
    else:
        heal.heal_attention_int16_noalloc(*args)
    status_ok()
    return to_np(out).astype(np.float64)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    d = dev()
    cases = [(make_inputs(B=4, Hq=32, Hkv=8, D=128, T=2048, seed=0), [2048, 1500, 64, 999]),
             (make_inputs(B=2, Hq=32, Hkv=8, D=128, T=1024, seed=7), [1024, 333])]
    for inputs, kv_len in cases:
        want = _run("workspace", inputs, kv_len, d)
        got = _run("noalloc", inputs, kv_len, d)
        q, qs, kq, kss, _, _ = inputs
        tol = tolerance(q, qs, kq, kss, kv_len, 128 ** -0.5, kq.shape[1])
        assert np.all(np.isfinite(got))
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= tol


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    d = dev()
    B, Hq, Hkv, D, Tmax = 256, 32, 8, 128, 64          # B*Hq*Tq = 8192 > 7939
    i16 = lambda *s: torch.zeros(*s, dtype=torch.int16, device=d)
    f32 = lambda *s: torch.zeros(*s, dtype=torch.float32, device=d)
    with pytest.raises(heal.HealError) as e:
        heal.heal_attention_int16_noalloc(i16(B, Hq, 1, D), f32(B, Hq, 1), i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax),
                                          i16(B, Hkv, Tmax, D), f32(B, Hkv, Tmax),
                                          torch.ones(B, dtype=torch.int32, device=d), 0.1, f32(B, Hq, 1, D))
    assert e.value.status == heal.HEAL_ERR_UNSUPPORTED


def test_noalloc_prefill_shape_matches_workspace_entry_point():
    # 4 query heads per KV head x 96 queries: the tcgen05 prefill kernel, whose byte planes
    # fit the fixed scratch at this size; the two entry points give the same bits
    d = dev()
    inputs = make_inputs(B=1, Hq=8, Hkv=2, D=128, T=192, Tq=96, seed=11)
    want = _run("workspace", inputs, [192], d)
    got = _run("noalloc", inputs, [192], d)
    assert np.array_equal(got, want)
