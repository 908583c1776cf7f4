"""GPU test of the reproducibility analogue and the FP32-pipeline baseline (the comparison of
the technical summary's Results: native BF16, full FP32 and HEAL-Full against a reference)
on a small random-init stack with 16-bit-representable weights.

Expected from the method: HEAL (INT16 Q/K/V, two-product GEMMs with FP32 accumulation and
no 16-bit store between kernels) stays near FP32 level against the FP64 truth -- the only
extra error is the INT16 rounding of Q/K/V, 2^-16 of each row's absmax -- while the plain
BF16 pipeline, which stores 16 bits at every kernel boundary, is orders of magnitude worse.
Bounds: FP32 logits within 1e-5 of FP64; HEAL within 2e-4 (INT16 Q/K/V through two layers
and the softmax); BF16's final-hidden MSE at least 100x HEAL's; no argmax flip for FP32 or
HEAL at any step whose FP64 top-2 margin exceeds 1e-3 of the largest logit.
"""
import pytest

import synthetic
from error_compensated_gemm_b200.study import reproducibility_study
from tests.gpu_helpers import dev

pytestmark = pytest.mark.gpu


def test_small_stack_heal_fp32_bf16_against_fp64():
    d = dev()
    cfg = synthetic.DecoderConfig(vocab=1000, hidden=256, heads=2, kv_heads=1, head_dim=128, ffn=512, layers=2,
                                  max_pos=256)
    res = reproducibility_study(d, cfg=cfg, prompt_len=64, steps=32, seed=20)
    p = res["pipelines"]
    print({k: {m: v[m] for m in ("logits_rel_err_max", "final_hidden_mse_mean", "argmax_flips", "tpot_ms")}
           for k, v in p.items()})
    assert p["fp32"]["logits_rel_err_max"] <= 1e-5
    assert p["heal"]["logits_rel_err_max"] <= 2e-4
    assert p["bf16_downcast"]["final_hidden_mse_mean"] >= 100 * p["heal"]["final_hidden_mse_mean"]
    assert p["bf16_downcast"]["logits_rel_err_mean"] >= 30 * p["heal"]["logits_rel_err_mean"]
    for name in ("fp32", "heal"):
        assert all(m < 1e-3 for m in p[name]["fp64_margin_at_flips"]), (name, p[name]["fp64_margin_at_flips"])
    for r in p.values():
        assert r["tpot_ms"] > 0
