// kv_quant.cu -- K4: per-(token, head) symmetric INT16 quantization of Q/K/V rows,
// written straight into the [B, H, Tmax, D] cache (gist.science technical summary,
// section 2.A: Q/K/V stored as INT16 at a 16-bit footprint).
//
// One group of L = D/8 lanes per row; each lane owns 8 consecutive values: one 16-byte
// (bf16) or two 16-byte (fp32) loads and one 16-byte int16 store.  The row absmax is a
// shuffle reduction inside the group.  Every decision is taken in FP32:
//   inv = 32767 / absmax (IEEE division), q = rint(x * inv) clamped to +-32767,
//   s = absmax / 32767; an all-zero row gives q = 0 and s = 0.
// HBM-bound: 2 (bf16) or 4 (fp32) bytes read and 2 bytes written per value.
#include <cuda_bf16.h>

#include "heal_internal.h"

namespace heal {

template <int L, bool BF16>
__global__ void __launch_bounds__(256) heal_kv_quant_kernel(const void* __restrict__ x, int B, int T, int H,
                                                            long long sb, long long st, long long sh,
                                                            int16_t* __restrict__ q, float* __restrict__ sc,
                                                            int Tmax, int t_off) {
  constexpr int D = 8 * L;
  constexpr int kRowsPerWarp = 32 / L;
  constexpr int kUnroll = 4;
  const int lane = threadIdx.x & 31;
  const int sub = lane % L;              // lane inside the row group
  const int grp = lane / L;              // row group inside the warp
  const long long rows = (long long)B * T * H;
  const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
  const long long warp_id = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long step = warps_total * kRowsPerWarp;

  for (long long r0 = warp_id * kRowsPerWarp * kUnroll; r0 < rows; r0 += step * kUnroll) {
    float v[kUnroll][8];
    long long rr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      rr[u] = r0 + (long long)u * kRowsPerWarp + grp;
      if (rr[u] < rows) {
        const long long r = rr[u];
        const int h = (int)(r % H);
        const long long bt = r / H;
        const int t = (int)(bt % T);
        const int b = (int)(bt / T);
        const long long off = b * sb + t * st + h * sh + sub * 8;
        if constexpr (BF16) {
          const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + off));
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            v[u][2 * j] = f.x;
            v[u][2 * j + 1] = f.y;
          }
        } else {
          const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + off);
          const float4 a = __ldcs(p), c = __ldcs(p + 1);
          v[u][0] = a.x; v[u][1] = a.y; v[u][2] = a.z; v[u][3] = a.w;
          v[u][4] = c.x; v[u][5] = c.y; v[u][6] = c.z; v[u][7] = c.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[u][j]));
#pragma unroll
      for (int o = L / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (rr[u] >= rows) continue;
      const long long r = rr[u];
      const int h = (int)(r % H);
      const long long bt = r / H;
      const int t = (int)(bt % T);
      const int b = (int)(bt / T);
      const long long row_out = ((long long)b * H + h) * Tmax + t_off + t;
      int qv[8];
      if (m > 0.0f) {
        const float inv = __fdiv_rn(32767.0f, m);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          int qi = __float2int_rn(__fmul_rn(v[u][j], inv));
          qv[j] = qi > 32767 ? 32767 : (qi < -32767 ? -32767 : qi);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) qv[j] = 0;
      }
      uint4 pk;
      pk.x = (uint32_t)(qv[0] & 0xFFFF) | ((uint32_t)qv[1] << 16);
      pk.y = (uint32_t)(qv[2] & 0xFFFF) | ((uint32_t)qv[3] << 16);
      pk.z = (uint32_t)(qv[4] & 0xFFFF) | ((uint32_t)qv[5] << 16);
      pk.w = (uint32_t)(qv[6] & 0xFFFF) | ((uint32_t)qv[7] << 16);
      *reinterpret_cast<uint4*>(q + row_out * D + sub * 8) = pk;
      if (sub == 0) sc[row_out] = m > 0.0f ? __fdiv_rn(m, 32767.0f) : 0.0f;
    }
  }
}

template <int L>
static cudaError_t launch_L(const void* x, int bf16, int B, int T, int H, long long sb, long long st, long long sh,
                            int16_t* q, float* sc, int Tmax, int t_off, int grid, cudaStream_t s) {
  if (bf16)
    heal_kv_quant_kernel<L, true><<<grid, 256, 0, s>>>(x, B, T, H, sb, st, sh, q, sc, Tmax, t_off);
  else
    heal_kv_quant_kernel<L, false><<<grid, 256, 0, s>>>(x, B, T, H, sb, st, sh, q, sc, Tmax, t_off);
  return cudaGetLastError();
}

heal_status_t kv_quant_launch(const void* x, int is_bf16, int B, int T, int H, int D, long long sb, long long st,
                              long long sh, int16_t* q, float* sc, int Tmax, int t_off, cudaStream_t s) {
  const long long rows = (long long)B * T * H;
  if (rows == 0) return HEAL_OK;
  const int sms = device_sm_count();
  if (sms <= 0) return HEAL_ERR_CUDA;
  const int L = D / 8;
  const long long rows_per_block = 8LL * (32 / L) * 4;   // 8 warps, kUnroll = 4
  long long grid = (rows + rows_per_block - 1) / rows_per_block;
  if (grid > (long long)sms * 8) grid = (long long)sms * 8;
  cudaError_t e;
  switch (L) {
    case 1: e = launch_L<1>(x, is_bf16, B, T, H, sb, st, sh, q, sc, Tmax, t_off, (int)grid, s); break;
    case 2: e = launch_L<2>(x, is_bf16, B, T, H, sb, st, sh, q, sc, Tmax, t_off, (int)grid, s); break;
    case 4: e = launch_L<4>(x, is_bf16, B, T, H, sb, st, sh, q, sc, Tmax, t_off, (int)grid, s); break;
    case 8: e = launch_L<8>(x, is_bf16, B, T, H, sb, st, sh, q, sc, Tmax, t_off, (int)grid, s); break;
    case 16: e = launch_L<16>(x, is_bf16, B, T, H, sb, st, sh, q, sc, Tmax, t_off, (int)grid, s); break;
    case 32: e = launch_L<32>(x, is_bf16, B, T, H, sb, st, sh, q, sc, Tmax, t_off, (int)grid, s); break;
    default: return HEAL_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

}  // namespace heal
