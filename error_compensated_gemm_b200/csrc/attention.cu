// attention.cu -- K5: decode attention on INT16 Q/K/V (gist.science technical summary,
// section 2.A, "Mechanism": the INT16 tensor is unpacked into two FP16 tensors for the
// attention contractions).
//
// Unpacking used here: q = 256*hi + lo with hi = q >> 8 in [-128, 127] and lo = q & 255
// in [0, 255].  Then, per (query row, token),
//     S_int = sum_d q_d k_d = 65536*S_hh + 256*S_x + S_ll
// with S_hh = sum qh*kh, S_x = sum (qh*kl + ql*kh), S_ll = sum ql*kl.  QK^T runs these four
// byte products on the integer tensor cores (mma.sync m16n8k32, signed hi bytes and
// unsigned lo bytes, exact int32 accumulation: for head_dim <= 128 no partial sum exceeds
// 2^24); the three sums are combined in int64.
//   logit = fp32( (double(S_int) * (double(s_q) * double(s_k))) * double(softmax_scale) )
// FP32 online softmax in base 2.  P is folded with the per-token V scale and a per-block
// power of two 2^E (chosen so the block's largest V scale times 2^E lies in [32, 64)),
// then split into FP16 P_hi and the FP16 residual r = P - P_hi; the byte-split V
// (hi = v >> 8, lo = v & 255, each an exact FP16 value) meets (256*P_hi, P_hi, 256*r, r) in
// four FP16 tensor-core products that accumulate into one FP32 accumulator:
// sum 256*hi*P + lo*P = v*P.  These are the two FP16 tensors the INT16 value is unpacked
// into for the floating-point contraction.
//
// Work decomposition: a persistent grid; CTA c owns the contiguous slice
// [total*c/grid, total*(c+1)/grid) of the sequence of (batch*kv_head, 64-token block)
// units.  Warp 4 streams 64-token K and V tiles with TMA (128-byte swizzle) into a
// two-stage ring (the K half of a stage is released after QK^T, the V half after PV);
// warps 0-3 each take 16 tokens of a tile with mma.sync (the decode GEMV shapes are far
// below a tcgen05 tile; the kernel is HBM-bound).  Every (CTA, kv head) segment leaves one
// partial (m, l, o) in the workspace; the combine kernel merges them in ascending token
// order.  The order is fixed, so results are identical from run to run.
#include <cuda_fp16.h>

#include <cmath>

#include "heal_internal.h"
#include "heal_ptx.cuh"

namespace heal {

namespace {

constexpr int kBlk = 64;          // tokens per pipeline stage
// K/V stages per CTA.  Two stages leave room for three CTAs (15 warps) per SM; on the
// 8 x 8192 x 8 x 128 decode cache three stages (two CTAs per SM) measured 9% slower and
// four or six (one CTA per SM) 44% slower: warps per SM matter more than ring depth here.
constexpr int kStages = 2;
constexpr int kMinBlocks = kStages <= 2 ? 3 : (kStages == 3 ? 2 : 1);   // CTAs per SM the ring allows
constexpr int kCompute = 4;       // compute warps, 16 tokens each per stage
constexpr int kAttnThreads = (kCompute + 1) * 32;
constexpr int kRows = 8;          // query rows per CTA: (Hq/Hkv) * Tq <= 8
constexpr int kMaxGrid = 1024;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
  const int16_t* q;
  const float* qs;
  const float* ks;
  const float* vs;
  const int32_t* kv_len;
  float* ws;
  long long* qk_out;
  float* out;
  int B, Hq, Hkv, G, Tq, R, Tmax, nblk, causal;
  float scale;
  long long total;  // B*Hkv*nblk
  int grid;
  unsigned int* status;
};

// -------- INT16 byte split into FP16 pairs (bit construction, exact) --------
// Two int16 values packed in x -> (lo0, lo1) and (hi0, hi1) as half2.
__device__ __forceinline__ uint32_t lo_pair(uint32_t x) {
  // 0x6400 | b is the FP16 value 1024 + b for b in [0, 1023]
  const uint32_t u = (x & 0x00FF00FFu) | 0x64006400u;
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&u), __half2half2(__ushort_as_half(0x6400)));
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t hi_pair(uint32_t x) {
  // (signed high byte + 128) in [0, 255]: XOR with 0x80, then the same construction
  const uint32_t u = ((x >> 8) & 0x00FF00FFu) ^ 0x64806480u;
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&u), __half2half2(__ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&h);   // 0x6480 = 1152 = 1024 + 128
}

// Bytes of two registers holding int16 pairs (x = (v0, v1), y = (v2, v3)):
// lo_bytes -> (v0 & 255, v1 & 255, v2 & 255, v3 & 255) as u8; hi_bytes -> their high bytes (s8).
__device__ __forceinline__ uint32_t lo_bytes(uint32_t x, uint32_t y) { return __byte_perm(x, y, 0x6420); }
__device__ __forceinline__ uint32_t hi_bytes(uint32_t x, uint32_t y) { return __byte_perm(x, y, 0x7531); }

// Exact integer MMA m16n8k32, s32 accumulate; A_U / B_U: the operand holds unsigned bytes.
template <bool A_U, bool B_U>
__device__ __forceinline__ void imma16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  if constexpr (!A_U && !B_U)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else if constexpr (!A_U && B_U)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else if constexpr (A_U && !B_U)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// x * 2^e for |e| <= 252 in two exact power-of-two steps (a single factor 2^e would
// overflow or underflow FP32 for |e| > 126, which extreme V scales can reach).
__device__ __forceinline__ float mul_pow2(float x, int e) {
  const int e1 = e / 2, e2 = e - e1;   // each in [-126, 126]
  return __fmul_rn(__fmul_rn(x, __int_as_float((127 + e1) << 23)), __int_as_float((127 + e2) << 23));
}

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kCompute * 32) : "memory"); }

__device__ __forceinline__ long long unit_begin(long long total, int grid, int c) {
  return (total * c) / grid;
}

// CTA whose slice contains unit u.
__device__ __forceinline__ int cta_of(long long u, long long total, int grid) {
  int c = (int)((u * grid) / total);
  while (c + 1 < grid && unit_begin(total, grid, c + 1) <= u) ++c;
  while (c > 0 && unit_begin(total, grid, c) > u) --c;
  return c;
}

// partial slot of (cta c, pair p) = c + p; layout: [R][D] o, then [R][2] (m, l)
__device__ __forceinline__ float* slot_ptr(float* ws, int c, int p, int R, int D) {
  return ws + (size_t)(c + p) * (size_t)R * (size_t)(D + 2);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, kMinBlocks) heal_attn_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                       const __grid_constant__ CUtensorMap tmV,
                                                                       const AttnArgs a) {
  constexpr int kBoxes = D / 64;                    // 64-dim (128-byte) boxes per row
  constexpr int kTileBytes = kBlk * D * 2;          // one of K / V
  constexpr int kStageBytes = 2 * kTileBytes;
  constexpr int kKSteps32 = D / 32;                 // k32 steps of the integer MMA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;                                                  // kStages x kStageBytes
  float* o_sm = reinterpret_cast<float*>(smem + kStages * kStageBytes);    // [kRows][D]
  float* ml_sm = o_sm + kRows * D;                                   // [kCompute][kRows][2]
  uint4* qf_sm = reinterpret_cast<uint4*>(ml_sm + kCompute * kRows * 2); // [kKSteps32][32 lanes]
  float* sc_sm = reinterpret_cast<float*>(qf_sm + kKSteps32 * 32);      // [kStages][K, V][kBlk]
  uint64_t* full = reinterpret_cast<uint64_t*>(sc_sm + kStages * 2 * kBlk);  // [S] K tile, [S] V tile + scales
  uint64_t* empty = full + 2 * kStages;                                // [S] K released, [S] V released
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + 2 * kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long u0 = unit_begin(a.total, a.grid, c), u1 = unit_begin(a.total, a.grid, c + 1);
  pdl_launch_dependents();   // the combine kernel may be scheduled; it waits for us

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2 * kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCompute);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCompute) {
    // ----------------------------- TMA producer -----------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int it = 0;
      for (long long u = u0; u < u1; ++u) {
        const int p = (int)(u / a.nblk), blk = (int)(u % a.nblk);
        const int b = p / a.Hkv;
        const int t0 = blk * kBlk;
        if (t0 >= __ldg(a.kv_len + b)) continue;
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        uint8_t* st = stages + s * kStageBytes;
        const int row = p * a.Tmax + t0;
        // K half: refilled as soon as the compute warps finish QK^T on the previous tile
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.status, 200)) break;
        mbar_arrive_expect_tx(&full[s], kTileBytes + kBlk * 4);
        bulk_load_1d(sc_sm + (s * 2 + 0) * kBlk, a.ks + (size_t)row, kBlk * 4, &full[s]);
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) tma_load_2d(st + bx * 8192, &tmK, &full[s], bx * 64, row);
        // V half and V scales
        if (!mbar_wait(&empty[kStages + s], ph ^ 1u, abort_flag, a.status, 202)) break;
        mbar_arrive_expect_tx(&full[kStages + s], kTileBytes + kBlk * 4);
        bulk_load_1d(sc_sm + (s * 2 + 1) * kBlk, a.vs + (size_t)row, kBlk * 4, &full[kStages + s]);
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx)
          tma_load_2d(st + kTileBytes + bx * 8192, &tmV, &full[kStages + s], bx * 64, row);
        ++it;
      }
      // no copy may still be in flight when the CTA exits
      for (int j = 0; j < kStages && j < it; ++j) {
        const int jt = it - 1 - j;
        volatile int dummy = 0;
        mbar_wait(&full[jt % kStages], (uint32_t)(jt / kStages) & 1u, &dummy, a.status, 201);
        mbar_wait(&full[kStages + jt % kStages], (uint32_t)(jt / kStages) & 1u, &dummy, a.status, 203);
      }
    }
    return;
  }

  // ------------------------------- compute warps -------------------------------
  // Fragment layouts (mma.sync, g = lane / 4, c = lane % 4):
  //   S^T = K Q^T with m16n8k32 integer MMAs: rows = this warp's 16 tokens, columns = the
  //   8 query rows.  C fragment of this lane: tokens g and g + 8, query rows 2c and 2c + 1.
  //   O^T = V^T P'^T with m16n8k16 FP16 MMAs: rows = 16 dims, columns = query rows; the
  //   lane holds dims g, g + 8 of query rows 2c, 2c + 1 (the same query rows as S^T).
  // Byte order inside the K dimension of the integer MMA: slot 4c + j of a 16-slot half
  // holds dim {2c, 2c + 1, 2c + 8, 2c + 9}[j] of that half; both operands use this order,
  // and a dot product does not depend on the order of its terms.
  const int R = a.R;
  const int g8 = lane >> 2;                   // token row (S^T) / dim row (O^T) / query of B fragments
  const int qc = 2 * (lane & 3);              // this lane's query rows qc, qc + 1
  float sq[2] = {0.0f, 0.0f};
  int pos[2] = {0, 0};
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};   // query rows qc + e
  float om[D / 16][4];                        // O^T accumulator (units of 2^E_run)
  int E_run = 0;                              // power of two folded into P (decreases only)
  bool have_E = false;
  int cur_p = -1, b = 0, hkv = 0, klen = 0;
  int it = 0;
  bool ok = true;

  auto finalize = [&](int p) {
    // per query row: the warp's maximum (replicated over g8) and its sum over all lanes
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[e];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      if (g8 == 0) {
        ml_sm[(warp * kRows + qc + e) * 2 + 0] = m_run[e];
        ml_sm[(warp * kRows + qc + e) * 2 + 1] = l;
      }
    }
    compute_bar();
    // query rows of this lane's O^T fragments: qc, qc + 1
    float f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = qc + h;
      float mx = -INFINITY;
      for (int w = 0; w < kCompute; ++w) mx = fmaxf(mx, ml_sm[(w * kRows + r) * 2]);
      const float mw = ml_sm[(warp * kRows + r) * 2];
      f[h] = (mw == -INFINITY) ? 0.0f : exp2f(mw - mx);
    }
    // O of this warp, scaled to the CTA max, in true units (x 2^-E_run), in place
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) om[dt][e] = __fmul_rn(mul_pow2(om[dt][e], -E_run), f[e & 1]);
    // sequential, fixed-order merge of the four warps through shared memory
    for (int w = 0; w < kCompute; ++w) {
      if (warp == w) {
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int d = dt * 16 + g8 + ((e >> 1) << 3);
            const int r = qc + (e & 1);
            float* dst = o_sm + r * D + d;
            const float v = (w == 0) ? om[dt][e] : __fadd_rn(*dst, om[dt][e]);
            if (w < kCompute - 1) {
              *dst = v;
            } else if (r < R) {
              slot_ptr(a.ws, c, p, R, D)[r * D + d] = v;
            }
          }
      }
      compute_bar();
    }
    if (warp == 0 && lane < R) {
      const int r = lane;
      float mx = -INFINITY;
      for (int w = 0; w < kCompute; ++w) mx = fmaxf(mx, ml_sm[(w * kRows + r) * 2]);
      float L = 0.0f;
      for (int w = 0; w < kCompute; ++w) {
        const float mw = ml_sm[(w * kRows + r) * 2];
        if (mw != -INFINITY) L = __fadd_rn(L, __fmul_rn(ml_sm[(w * kRows + r) * 2 + 1], exp2f(mw - mx)));
      }
      float* sl = slot_ptr(a.ws, c, p, R, D) + R * D;
      sl[2 * r] = mx;
      sl[2 * r + 1] = L;
    }
    compute_bar();
  };

  for (long long u = u0; u < u1 && ok; ++u) {
    const int p = (int)(u / a.nblk), blk = (int)(u % a.nblk);
    if (p != cur_p) {
      if (cur_p >= 0) finalize(cur_p);
      cur_p = p;
      b = p / a.Hkv;
      hkv = p % a.Hkv;
      klen = __ldg(a.kv_len + b);
      // query row r = tq * G + g of this kv head  ->  head hkv*G + g, query tq
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = qc + e;
        const bool real = r < R;
        const int tq = real ? r / a.G : 0, gq = real ? r % a.G : 0;
        sq[e] = real ? __ldg(a.qs + ((long long)(b * a.Hq + hkv * a.G + gq) * a.Tq + tq)) : 0.0f;
        pos[e] = klen - a.Tq + tq;
      }
      // B fragments of Q^T (query row g8), byte-split, one table per CTA:
      // entry [s][lane] = (hi slots 0-15, hi slots 16-31, lo slots 0-15, lo slots 16-31)
      if (warp == 0) {
        const int r = g8;
        const bool real = r < R;
        const int tq = real ? r / a.G : 0, gq = real ? r % a.G : 0;
        const long long qrow = ((long long)(b * a.Hq + hkv * a.G + gq) * a.Tq + tq);
#pragma unroll
        for (int s32 = 0; s32 < kKSteps32; ++s32) {
          uint32_t w[4] = {0u, 0u, 0u, 0u};
          if (real) {
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.q + qrow * D + s32 * 32 + qc);
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = __ldg(qp + 4 * i);   // dims 32s + 8i + 2c, +1
          }
          qf_sm[s32 * 32 + lane] = make_uint4(hi_bytes(w[0], w[1]), hi_bytes(w[2], w[3]), lo_bytes(w[0], w[1]),
                                              lo_bytes(w[2], w[3]));
        }
      }
      compute_bar();
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        m_run[e] = -INFINITY;
        l_run[e] = 0.0f;
      }
      E_run = 0;
      have_E = false;
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) om[dt][e] = 0.0f;
    }
    const int t0 = blk * kBlk;
    if (t0 >= klen) continue;
    const int s = it % kStages;
    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
    ++it;
    if (!mbar_wait(&full[s], ph, abort_flag, a.status, 210)) {
      ok = false;
      break;
    }
    const uint32_t kst = smem_u32(stages + s * kStageBytes);
    const uint32_t vst = kst + kTileBytes;
    const float* sks = sc_sm + (s * 2 + 0) * kBlk;   // K scales of this block's 64 tokens
    const float* svs = sc_sm + (s * 2 + 1) * kBlk;   // V scales
    const int tw = warp * 16;                 // this warp's first token inside the tile

    // ---- exact S^T = K Q^T on the byte-split operands (integer tensor cores) ----
    // S_x in two accumulators (kh.ql and kl.qh) so no MMA chain is longer than the k32 steps
    int shh[4] = {0, 0, 0, 0}, sxa[4] = {0, 0, 0, 0}, sxb[4] = {0, 0, 0, 0}, sll[4] = {0, 0, 0, 0};
#pragma unroll
    for (int s32 = 0; s32 < kKSteps32; ++s32) {
      const uint4 qf = qf_sm[s32 * 32 + lane];
      uint32_t r[2][4];                       // [token half][16-byte chunk 4*s32 + i]
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const int trow = tw + th * 8 + (lane & 7);
        const int ch = 4 * s32 + (lane >> 3);   // 16-byte chunk of the K row
        const uint32_t addr = kst + (ch >> 3) * 8192 + trow * 128 + ((((ch & 7) ^ (trow & 7))) << 4);
        ldsm_x4(addr, r[th][0], r[th][1], r[th][2], r[th][3]);
      }
      // A fragments: a0 token g8 slots 0-15, a1 token g8+8, a2 token g8 slots 16-31, a3 token g8+8
      const uint32_t ah0 = hi_bytes(r[0][0], r[0][1]), ah1 = hi_bytes(r[1][0], r[1][1]);
      const uint32_t ah2 = hi_bytes(r[0][2], r[0][3]), ah3 = hi_bytes(r[1][2], r[1][3]);
      const uint32_t al0 = lo_bytes(r[0][0], r[0][1]), al1 = lo_bytes(r[1][0], r[1][1]);
      const uint32_t al2 = lo_bytes(r[0][2], r[0][3]), al3 = lo_bytes(r[1][2], r[1][3]);
      imma16832<false, false>(shh, ah0, ah1, ah2, ah3, qf.x, qf.y);
      imma16832<false, true>(sxa, ah0, ah1, ah2, ah3, qf.z, qf.w);
      imma16832<true, false>(sxb, al0, al1, al2, al3, qf.x, qf.y);
      imma16832<true, true>(sll, al0, al1, al2, al3, qf.z, qf.w);
    }
    // every ldmatrix of the K tile has been consumed by the MMAs above and the K scales
    // this lane needs are copied to registers: release the K half now, before the logit
    // arithmetic, so the producer can refill it sooner
    float skr[2];
#pragma unroll
    for (int th = 0; th < 2; ++th) skr[th] = sks[tw + th * 8 + g8];
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    float x[2][2];                            // [token half][query e]: logit * log2(e)
#pragma unroll
    for (int th = 0; th < 2; ++th) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * th + e;
        const int t = t0 + tw + th * 8 + g8;
        const int r = qc + e;
        const long long S = ((long long)shh[i] << 16) + (((long long)sxa[i] + (long long)sxb[i]) << 8) +
                            (long long)sll[i];
        const bool real = r < R;
        const bool vis = real && t < klen && (!a.causal || t <= pos[e]);
        float xv;
        if (!real) {
          xv = 0.0f;                          // padding query row: finite, never written
        } else if (!vis) {
          xv = -INFINITY;
        } else {
          const double coef = (double)sq[e] * (double)skr[th];
          const float lg = (float)(((double)S * coef) * (double)a.scale);
          xv = __fmul_rn(lg, kLog2e);
          if (a.qk_out) {
            const int tq = r / a.G, gq = r % a.G;
            a.qk_out[((long long)(b * a.Hq + hkv * a.G + gq) * a.Tq + tq) * a.Tmax + t] = S;
          }
        }
        x[th][e] = xv;
      }
    }

    if (!mbar_wait(&full[kStages + s], ph, abort_flag, a.status, 211)) {
      ok = false;
      break;
    }

    // ---- online softmax (base 2) of query rows qc, qc + 1 over this warp's tokens ----
    float alpha[2], pv[2][2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float bm = fmaxf(x[0][e], x[1][e]);
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
      const float m_new = fmaxf(m_run[e], bm);
      if (m_new == -INFINITY) {
        alpha[e] = 1.0f;
        pv[0][e] = pv[1][e] = 0.0f;
      } else {
        alpha[e] = (m_run[e] == -INFINITY) ? 0.0f : exp2f(m_run[e] - m_new);
#pragma unroll
        for (int th = 0; th < 2; ++th) pv[th][e] = (x[th][e] == -INFINITY) ? 0.0f : exp2f(x[th][e] - m_new);
      }
      l_run[e] = __fadd_rn(__fmul_rn(l_run[e], alpha[e]), __fadd_rn(pv[0][e], pv[1][e]));
      m_run[e] = m_new;
    }
    // power of two for this block: the largest visible V scale times 2^E in [32, 64)
    // (V scales are non-negative, so their bit patterns order like the floats: one
    // warp-wide integer max gives the block maximum)
    float smax;
    {
      const int ta = t0 + lane, tb = t0 + 32 + lane;
      unsigned int um = 0u;
      if (ta < klen) um = __float_as_uint(svs[lane]);
      if (tb < klen) um = max(um, __float_as_uint(svs[32 + lane]));
      smax = __uint_as_float(__reduce_max_sync(0xffffffffu, um));
    }
    float escale = 1.0f;                       // 2^(E_new - E_run) applied to O
    if (smax > 0.0f) {
      const int E_blk = 5 - ilogbf(smax);
      if (!have_E) {
        E_run = E_blk;
        have_E = true;
      } else if (E_blk < E_run) {
        escale = ldexpf(1.0f, E_blk - E_run);
        E_run = E_blk;
      }
    }
    // rescale O^T columns qc, qc + 1 (this lane's own query rows)
    const float a0 = __fmul_rn(alpha[0], escale);
    const float a1 = __fmul_rn(alpha[1], escale);
    if (!__all_sync(0xffffffffu, a0 == 1.0f && a1 == 1.0f)) {
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        om[dt][0] = __fmul_rn(om[dt][0], a0);
        om[dt][1] = __fmul_rn(om[dt][1], a1);
        om[dt][2] = __fmul_rn(om[dt][2], a0);
        om[dt][3] = __fmul_rn(om[dt][3], a1);
      }
    }

    // ---- P' = P * s_v * 2^E (S^T layout), moved to the B layout of PV: lane (g8, c)
    // needs tokens 2c, 2c + 1, 2c + 8, 2c + 9 of query row g8.  Token 2c + j lives in lane
    // 4 * (2c + j) + g8 / 2 (halves th = 0 / 1 for +0 / +8), query row g8 in its slot g8 & 1.
    float pp[2][2];
#pragma unroll
    for (int th = 0; th < 2; ++th) {
      const int t = t0 + tw + th * 8 + g8;
      const float svt = mul_pow2(svs[t - t0], E_run);   // s_v * 2^E, in [0, 64)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float sv = (pv[th][e] != 0.0f) ? svt : 0.0f;
        pp[th][e] = __fmul_rn(pv[th][e], sv);
      }
    }
    float pt[2][2];                            // [token half][j]: P' of token 8*half + 2c + j, query g8
    {
      const int cq = lane & 3;
      const bool odd = (g8 & 1) != 0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int src = 4 * (2 * cq + j) + (g8 >> 1);
#pragma unroll
        for (int th = 0; th < 2; ++th) {
          const float v0 = __shfl_sync(0xffffffffu, pp[th][0], src);
          const float v1 = __shfl_sync(0xffffffffu, pp[th][1], src);
          pt[th][j] = odd ? v1 : v0;
        }
      }
    }
    // FP16 P_hi and residual r = P' - P_hi: B fragments of PV
    uint32_t ph_[2], pr_[2], ph256[2], pr256[2];
#pragma unroll
    for (int th = 0; th < 2; ++th) {
      const __half2 h = __floats2half2_rn(pt[th][0], pt[th][1]);
      const float2 hf = __half22float2(h);
      const __half2 rr = __floats2half2_rn(__fsub_rn(pt[th][0], hf.x), __fsub_rn(pt[th][1], hf.y));
      const __half2 k256 = __half2half2(__ushort_as_half(0x5C00));   // 256.0
      const __half2 h256 = __hmul2(h, k256), r256 = __hmul2(rr, k256); // exact: powers of two
      ph_[th] = *reinterpret_cast<const uint32_t*>(&h);
      pr_[th] = *reinterpret_cast<const uint32_t*>(&rr);
      ph256[th] = *reinterpret_cast<const uint32_t*>(&h256);
      pr256[th] = *reinterpret_cast<const uint32_t*>(&r256);
    }

    // ---- O^T += V^T P'^T  (256*hi*P + lo*P with P = P_hi + r) ----
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
      const int mi = lane >> 3;
      const int trow = tw + ((mi >> 1) << 3) + (lane & 7);
      const int ch = 2 * dt + (mi & 1);
      const uint32_t addr = vst + (ch >> 3) * 8192 + trow * 128 + ((((ch & 7) ^ (trow & 7))) << 4);
      uint32_t r0, r1, r2, r3;
      ldsm_x4_t(addr, r0, r1, r2, r3);
      const uint32_t h0 = hi_pair(r0), h1 = hi_pair(r1), h2 = hi_pair(r2), h3 = hi_pair(r3);
      const uint32_t l0 = lo_pair(r0), l1 = lo_pair(r1), l2 = lo_pair(r2), l3 = lo_pair(r3);
      mma16816(om[dt], h0, h1, h2, h3, ph256[0], ph256[1]);
      mma16816(om[dt], l0, l1, l2, l3, ph_[0], ph_[1]);
      mma16816(om[dt], h0, h1, h2, h3, pr256[0], pr256[1]);
      mma16816(om[dt], l0, l1, l2, l3, pr_[0], pr_[1]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[kStages + s]);
  }
  if (!ok) return;   // a wait gave up: the status word is set; leave without a partial
  if (cur_p >= 0) finalize(cur_p);
}

// out[b, hq, tq, :] = sum_c o_c 2^(m_c - M) / sum_c l_c 2^(m_c - M), c ascending.
// The partials of kCombBatch CTAs are requested together (independent loads) and then
// applied one by one in ascending CTA order, so the sums are the same as a one-at-a-time
// loop while the number of dependent memory round trips drops by kCombBatch.
constexpr int kCombBatch = 8;
template <int D>
__global__ void __launch_bounds__(D) heal_attn_combine_kernel(const AttnArgs a) {
  pdl_wait_prerequisites();             // the decode kernel that wrote the partials has completed
  const int pr = blockIdx.x;            // (pair, row)
  const int p = pr / a.R, r = pr % a.R;
  const int d = threadIdx.x;
  const long long ufirst = (long long)p * a.nblk, ulast = ufirst + a.nblk - 1;
  const int c0 = cta_of(ufirst, a.total, a.grid), c1 = cta_of(ulast, a.total, a.grid);
  float M = -INFINITY;
  for (int cb = c0; cb <= c1; cb += kCombBatch) {
    float m[kCombBatch];
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t)
      m[t] = (cb + t <= c1) ? slot_ptr(a.ws, cb + t, p, a.R, D)[a.R * D + 2 * r] : -INFINITY;
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) M = fmaxf(M, m[t]);
  }
  float L = 0.0f, O = 0.0f;
  for (int cb = c0; cb <= c1; cb += kCombBatch) {
    float m[kCombBatch], l[kCombBatch], o[kCombBatch];
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) {
      const bool in = cb + t <= c1;
      const float* sl = slot_ptr(a.ws, in ? cb + t : c0, p, a.R, D);
      m[t] = in ? sl[a.R * D + 2 * r] : -INFINITY;
      l[t] = in ? sl[a.R * D + 2 * r + 1] : 0.0f;
      o[t] = in ? sl[r * D + d] : 0.0f;
    }
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) {
      if (m[t] == -INFINITY) continue;
      const float f = exp2f(m[t] - M);
      L = __fadd_rn(L, __fmul_rn(l[t], f));
      O = __fadd_rn(O, __fmul_rn(o[t], f));
    }
  }
  const int b = p / a.Hkv, hkv = p % a.Hkv;
  const int tq = r / a.G, g = r % a.G;
  // a query with no visible token (causal, kv_len < Tq) gets zeros
  a.out[(((long long)(b * a.Hq + hkv * a.G + g) * a.Tq + tq) * D) + d] = L > 0.0f ? __fdiv_rn(O, L) : 0.0f;
}

template <int D>
constexpr int attn_smem_bytes() {
  return kStages * (2 * kBlk * D * 2) + kRows * D * 4 + kCompute * kRows * 2 * 4 + (D / 32) * 32 * 16 +
         kStages * 2 * kBlk * 4 + 2 * 2 * kStages * 8 + 32 + 1024;
}

}  // namespace

size_t attention_workspace_bytes(int B, int Hq, int Tq, int Tmax) {
  (void)Tmax;
  // slots <= grid + B*Hkv; slot = R*(D+2) floats with R*Hkv = Hq*Tq, R <= 8, D <= 128
  return ((size_t)kMaxGrid * kRows + (size_t)B * Hq * Tq) * 130u * sizeof(float);
}

heal_status_t attention_launch(const int16_t* q, const float* qs, const int16_t* k, const float* ks,
                               const int16_t* v, const float* vs, int B, int Hq, int Hkv, int D, int Tq,
                               const int32_t* kv_len, int Tmax, float scale, int causal, float* out, void* ws,
                               size_t ws_bytes, int64_t* qk_out, cudaStream_t stream) {
  const int G = Hq / Hkv;
  const int R = G * Tq;
  if (R > kRows) return HEAL_ERR_UNSUPPORTED;
  const long long rows_total = (long long)B * Hkv * Tmax;
  if (rows_total >= (1LL << 31)) return HEAL_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return HEAL_ERR_CUDA;
  AttnArgs a{};
  a.q = q;
  a.qs = qs;
  a.ks = ks;
  a.vs = vs;
  a.kv_len = kv_len;
  a.ws = static_cast<float*>(ws);
  a.qk_out = reinterpret_cast<long long*>(qk_out);
  a.out = out;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = G;
  a.Tq = Tq;
  a.R = R;
  a.Tmax = Tmax;
  a.nblk = Tmax / kBlk;
  a.causal = causal;
  a.scale = scale;
  a.total = (long long)B * Hkv * a.nblk;
  // once per device: opt in to the large shared-memory carve-out (the occupancy query
  // depends on it), then ask how many CTAs fit per SM
  static int per_sm_cache[64][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HEAL_ERR_CUDA;
  const int di = (D == 128) ? 0 : 1;
  int per_sm = per_sm_cache[dev][di];
  if (per_sm == 0) {
    if (cudaFuncSetAttribute(heal_attn_decode_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem_bytes<128>()) != cudaSuccess ||
        cudaFuncSetAttribute(heal_attn_decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem_bytes<64>()) != cudaSuccess)
      return HEAL_ERR_CUDA;
    if (D == 128)
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, heal_attn_decode_kernel<128>, kAttnThreads,
                                                    attn_smem_bytes<128>());
    else
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, heal_attn_decode_kernel<64>, kAttnThreads,
                                                    attn_smem_bytes<64>());
    if (per_sm < 1) per_sm = 1;
    per_sm_cache[dev][di] = per_sm;
  }
  long long grid = (long long)sms * per_sm;
  if (grid > kMaxGrid) grid = kMaxGrid;
  if (grid > a.total) grid = a.total;
  a.grid = (int)grid;
  a.status = device_status_ptr();
  if ((size_t)(a.grid + (long long)B * Hkv) * (size_t)R * (size_t)(D + 2) * sizeof(float) > ws_bytes)
    return HEAL_ERR_INVALID_ARGUMENT;

  CUtensorMap tk{}, tv{};
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows_total};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, kBlk};
  const cuuint32_t es[2] = {1, 1};
  if (!encode_tensor_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<int16_t*>(k), dims, strides, box, es,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return HEAL_ERR_CUDA;
  if (!encode_tensor_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<int16_t*>(v), dims, strides, box, es,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return HEAL_ERR_CUDA;
  cudaError_t e;
  if (D == 128) {
    heal_attn_decode_kernel<128><<<a.grid, kAttnThreads, attn_smem_bytes<128>(), stream>>>(tk, tv, a);
    e = launch_pdl(heal_attn_combine_kernel<128>, dim3(B * Hkv * R), dim3(128), 0, stream, a);
  } else {
    heal_attn_decode_kernel<64><<<a.grid, kAttnThreads, attn_smem_bytes<64>(), stream>>>(tk, tv, a);
    e = launch_pdl(heal_attn_combine_kernel<64>, dim3(B * Hkv * R), dim3(64), 0, stream, a);
  }
  if (e != cudaSuccess) return HEAL_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

}  // namespace heal
