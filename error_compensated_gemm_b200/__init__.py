"""error_compensated_gemm_b200 -- B200 (sm_100a) hot path of HEAL.

HEAL ("Demystifying Numerical Instability in LLM Inference ... with HEAL", arXiv
2606.21023) computes FP32-accurate GEMMs on 16-bit tensor cores by splitting each FP32
operand into a 16-bit value and a 16-bit residual, and stores Q/K/V as INT16 that is
unpacked into exact FP16 pairs for attention.  The kernels live in libheal.so (C ABI,
include/heal.h); this package is its Python binding.  Importing it does not load the
library; the first call does, and fails loudly if the CUDA extension is missing.
"""
from ._binding import (  # noqa: F401
    EXPORTED, HEAL_ERR_CUDA, HEAL_ERR_INVALID_ARGUMENT, HEAL_ERR_TIMEOUT, HEAL_ERR_UNSUPPORTED, HEAL_OK,
    SPLIT_BF16, SPLIT_FP16_S11, TILE_128x128, TILE_256x256_PAIR, TILE_AUTO, TILE_SKINNY_CHAIN, TILE_SKINNY_FULLK, TILE_SKINNY_SPLITK, GemmOpts, HealError,
    gemm_opts, heal_attention_int16, heal_attention_int16_noalloc, heal_attention_workspace_bytes,
    heal_attention_workspace_bytes_gqa, heal_gemm_compensated,
    heal_gemm_workspace_bytes, heal_get_device_status, heal_kv_quantize_int16, heal_split, heal_version, lib,
    status_string, heal_embedding_gather, heal_rmsnorm, heal_rope, heal_swiglu, heal_add, heal_argmax,
    heal_probe_wait_timeout, heal_heads_to_rows)

__version__ = "0.1.0"
