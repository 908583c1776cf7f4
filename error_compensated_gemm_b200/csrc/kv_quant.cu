// kv_quant.cu -- K4: per-(token, head) symmetric INT16 quantization of Q/K/V rows,
// written straight into the [B, H, Tmax, D] cache (gist.science technical summary,
// section 2.A: Q/K/V stored as INT16 at a 16-bit footprint).
//
// A warp takes one unit at a time: a token (b, t) and a group of up to 4 * 32/L of its H
// head rows (all of them when H is small; several units per token when H is large, so that
// a step with few tokens, such as one decode query, still spreads over many warps), in
// passes of 32/L rows, one group of L = D/8 lanes per row; each lane owns 8 consecutive values: one 16-byte
// (bf16) or two 16-byte (fp32) streaming loads and one 16-byte int16 store.  The row
// absmax is a shuffle reduction inside the group.  Every decision is taken in FP32:
//   inv = 32767 / absmax (IEEE division), q = rint(x * inv) clamped to +-32767,
//   s = absmax / 32767; an all-zero row gives q = 0 and s = 0.
// A unit's divisions (two per row) are spread over the warp's lanes, one division
// sequence per 16 rows, and rint is an FP32 add of 1.5 * 2^23 whose low 16 bits are
// the code: the per-value work is a multiply, an add and half a byte permute.
// HBM-bound: 2 (bf16) or 4 (fp32) bytes read and 2 bytes written per value.
#include <cuda_bf16.h>

#include "heal_internal.h"
#include "heal_ptx.cuh"

namespace heal {

template <int L, bool BF16>
__global__ void __launch_bounds__(256, 4) heal_kv_quant_kernel(const void* __restrict__ x, int B, int T, int H,
                                                            long long sb, long long st, long long sh,
                                                            int16_t* __restrict__ q, float* __restrict__ sc,
                                                            int Tmax, int t_off, unsigned int* status) {
  // programmatic dependent launch: the next kernel may be scheduled now; the preceding one
  // (which may write x or read the cache) finishes before the first global access here
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  constexpr int D = 8 * L;
  constexpr int kRowsPerPass = 32 / L;      // (token, head) rows one warp covers per pass
  constexpr int kUnroll = 4;                // passes whose loads are in flight together
  const int lane = threadIdx.x & 31;
  const int sub = lane % L;                 // lane inside the row group
  const int grp = lane / L;                 // row group inside the warp
  const int tokens = B * T;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int warp_id = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);

  // one warp per (token, head group) unit; the group's rows in kUnroll passes of kRowsPerPass
  constexpr int kGroupRows = kRowsPerPass * kUnroll;
  const int hgroups = (H + kGroupRows - 1) / kGroupRows;
  const long long units = (long long)tokens * hgroups;
  for (long long un = warp_id; un < units; un += warps_total) {
    const int bt = (int)(un / hgroups), hg = (int)(un - (long long)bt * hgroups);
    const int b = bt / T, t = bt - b * T;
    const char* xrow = static_cast<const char*>(x) + (size_t)(b * sb + (long long)t * st) * (BF16 ? 2 : 4);
    {
      const int h0 = hg * kGroupRows;
      // all loads of the pass group first, kept as raw words (4 registers per 16 bytes)
      uint4 raw[kUnroll][BF16 ? 1 : 2];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int h = h0 + u * kRowsPerPass + grp;
        if (h < H) {
          if constexpr (BF16) {
            raw[u][0] = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(xrow) +
                                                              (size_t)h * sh + sub * 8));
          } else {
            const uint4* pf = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(xrow) + (size_t)h * sh +
                                                             sub * 8);
            raw[u][0] = __ldcs(pf);
            raw[u][1] = __ldcs(pf + 1);
          }
        } else {
          raw[u][0] = make_uint4(0, 0, 0, 0);
          if constexpr (!BF16) raw[u][1] = make_uint4(0, 0, 0, 0);
        }
      }
      // widen to FP32 and take each row's absmax (a shuffle reduction inside the group)
      float vv[kUnroll][8];
      float mrow[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if constexpr (BF16) {
          // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 pattern
          const uint32_t w[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            vv[u][2 * j] = __uint_as_float(w[j] << 16);
            vv[u][2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
          }
        } else {
          const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                 raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
#pragma unroll
          for (int j = 0; j < 8; ++j) vv[u][j] = __uint_as_float(w[j]);
        }
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(vv[u][j]));
#pragma unroll
        for (int o = L / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        mrow[u] = m;
      }
      // The unit's IEEE divisions, spread over the lanes instead of repeated in every lane
      // of a row group: task j = 2 * row + kind, kind 0 -> inv = 32767 / absmax, kind 1 ->
      // s = absmax / 32767 (row = u * kRowsPerPass + group; 0 for an all-zero row).
      constexpr int kTasks = 2 * kGroupRows;
      constexpr int kSeq = (kTasks + 31) / 32;
      float res[kSeq];
#pragma unroll
      for (int sq = 0; sq < kSeq; ++sq) {
        const int j = sq * 32 + lane;
        const int row = (j >> 1) < kGroupRows ? (j >> 1) : kGroupRows - 1;
        const int ur = row / kRowsPerPass, gr = row % kRowsPerPass;
        float mm = 0.0f;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const float tv = __shfl_sync(0xffffffffu, mrow[u], gr * L);
          if (u == ur) mm = tv;
        }
        const bool kind_s = (j & 1) != 0;
        res[sq] = mm > 0.0f ? __fdiv_rn(kind_s ? mm : 32767.0f, kind_s ? 32767.0f : mm) : 0.0f;
        const int h = h0 + row;
        if (kind_s && j < kTasks && h < H) {
          const long long row_out = ((long long)b * H + h) * Tmax + t_off + t;
          if (HEAL_DCHECK(row_out < (long long)B * H * Tmax && t_off + t < Tmax, status, 401)) sc[row_out] = res[sq];
        }
      }
      // Codes.  |x * inv| <= 32767 (1 + 2^-24) rounded, so rint never leaves [-32767, 32767]
      // and the clamp of the definition is never active.  rint (ties to even) is taken by
      // adding 1.5 * 2^23: the sum lies in [2^23, 2^24), where the FP32 spacing is 1, so its
      // round-to-nearest-even is 1.5 * 2^23 + rint(y) and the low 16 bits of its pattern are
      // rint(y) in two's complement.  (A row with absmax 0 has inv = 0 and codes 0.)
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int jt = 2 * (u * kRowsPerPass + grp);   // the task holding this row's inv
        float inv = 0.0f;
#pragma unroll
        for (int sq = (2 * u * kRowsPerPass) / 32; sq <= (2 * (u + 1) * kRowsPerPass - 1) / 32 && sq < kSeq; ++sq) {
          const float tv = __shfl_sync(0xffffffffu, res[sq], jt & 31);
          if ((jt >> 5) == sq) inv = tv;
        }
        const int h = h0 + u * kRowsPerPass + grp;
        if (h >= H) continue;
        const long long row_out = ((long long)b * H + h) * Tmax + t_off + t;
        uint32_t c[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = __float_as_uint(__fadd_rn(__fmul_rn(vv[u][j], inv), 12582912.0f));
        uint4 pk;
        pk.x = __byte_perm(c[0], c[1], 0x5410);
        pk.y = __byte_perm(c[2], c[3], 0x5410);
        pk.z = __byte_perm(c[4], c[5], 0x5410);
        pk.w = __byte_perm(c[6], c[7], 0x5410);
        if (HEAL_DCHECK(row_out < (long long)B * H * Tmax && t_off + t < Tmax, status, 400))
          __stcs(reinterpret_cast<uint4*>(q + row_out * D + sub * 8), pk);
      }
    }
  }
}

template <int L>
static cudaError_t launch_L(const void* x, int bf16, int B, int T, int H, long long sb, long long st, long long sh,
                            int16_t* q, float* sc, int Tmax, int t_off, int grid, cudaStream_t s) {
  if (bf16)
    return launch_pdl(heal_kv_quant_kernel<L, true>, dim3(grid), dim3(256), 0, s, x, B, T, H, sb, st, sh, q, sc, Tmax,
                      t_off, device_status_ptr());
  return launch_pdl(heal_kv_quant_kernel<L, false>, dim3(grid), dim3(256), 0, s, x, B, T, H, sb, st, sh, q, sc, Tmax,
                    t_off, device_status_ptr());
}

heal_status_t kv_quant_launch(const void* x, int is_bf16, int B, int T, int H, int D, long long sb, long long st,
                              long long sh, int16_t* q, float* sc, int Tmax, int t_off, cudaStream_t s) {
  const long long rows = (long long)B * T * H;
  if (rows == 0) return HEAL_OK;
  if ((long long)B * T >= (1LL << 31)) return HEAL_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return HEAL_ERR_CUDA;
  const int L = D / 8;
  const long long tokens = (long long)B * T;
  const long long group_rows = 128 / L;                  // head rows per warp unit (4 passes of 32/L)
  const long long units = tokens * ((H + group_rows - 1) / group_rows);
  long long grid = (units + 7) / 8;                      // 8 warps per block, one unit each
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
