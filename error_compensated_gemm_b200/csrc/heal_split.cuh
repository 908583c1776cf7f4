// heal_split.cuh -- the hi/lo residual split of two FP32 values (gist.science technical
// summary, section 2.B: a primary 16-bit value plus a residual error term).
//   FMT 0 (FP16, residual scaled by 2^11): hi = fp16_rn(x), lo = fp16_rn((x - hi) * 2^11)
//   FMT 1 (BF16, unscaled residual):       hi = bf16_rn(x), lo = bf16_rn(x - hi)
// x - hi is exact in FP32; every rounding is to nearest-even and nothing is contracted.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace heal {

template <int FMT>
__device__ __forceinline__ uint32_t split2(float a, float b, uint32_t& lo_out) {
  if constexpr (FMT == 0) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(__fmul_rn(__fsub_rn(a, hf.x), 2048.0f),
                                        __fmul_rn(__fsub_rn(b, hf.y), 2048.0f));
    lo_out = *reinterpret_cast<const uint32_t*>(&l);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(a, hf.x), __fsub_rn(b, hf.y));
    lo_out = *reinterpret_cast<const uint32_t*>(&l);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

}  // namespace heal
