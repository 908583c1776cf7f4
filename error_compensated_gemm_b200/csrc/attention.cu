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
// 2^24); the test hook receives their exact int64 combination.  The logit, in log2 units:
//   x = fp32( fp32(fp32(S_int) * s_k) * fp32(fp32(s_q * softmax_scale) * log2(e)) )
// with fp32(S_int) = fp32(65536*S_hh + fp32(256*S_x + S_ll)) (S_hh exact in FP32; two
// roundings), as in the prefill kernel.  FP32 online softmax in base 2 (2^x by
// ex2.approx, as in the prefill kernel).  P is folded with
// the per-token V scale and a per-block power of two 2^E (chosen so the block's largest V
// scale times 2^E lies in [32, 64)), then split into FP16 P_hi and the FP16 residual
// r = P - P_hi; the byte-split V
// (hi = v >> 8, lo = v & 255, each an exact FP16 value) meets (256*P_hi, P_hi, 256*r, r) in
// four FP16 tensor-core products that accumulate into one FP32 accumulator:
// sum 256*hi*P + lo*P = v*P.  These are the two FP16 tensors the INT16 value is unpacked
// into for the floating-point contraction.
//
// Work decomposition: a persistent grid (three CTAs per SM); CTA c owns the contiguous
// slice [total*c/grid, total*(c+1)/grid) of the sequence of (batch*kv_head, 64-token
// block) units.  Warp roles: a TMA producer streams 64-token K and V tiles (128-byte
// swizzle) into a two-stage ring; four QK warps take 16 tokens each (exact S^T on the
// integer tensor cores, logits, the block's softmax step with the row maximum shared by
// the four warps, P' split into FP16 parts and written in the PV operand layout); four PV
// warps each own a quarter of the dims of O and add V^T P'^T over the block's 64 tokens.
// The two groups work on consecutive blocks at the same time.  mma.sync rather than
// tcgen05: the decode shapes (<= 8 query rows per KV head) are far below a tcgen05 tile
// and the kernel is HBM-bound.  Every (CTA, kv head) segment leaves one partial (m, l, o)
// in the workspace; the combine kernel merges them in ascending token order.  The order
// is fixed, so results are identical from run to run.
#include <cuda_fp16.h>

#include <cmath>

#include "heal_internal.h"
#include "heal_ptx.cuh"

namespace heal {

namespace {

constexpr int kBlk = 64;          // tokens per pipeline stage
// Warp roles per CTA: kQK warps for QK^T and the softmax step (16 tokens each), kPV warps
// for PV (D/4 dims each), one TMA producer.  Two K/V stages per CTA, three CTAs per SM
// (24 compute warps and six stages per SM: the consumers' instruction streams are latency
// bound, so more warps per SM keep more K/V bytes moving).
constexpr int kQK = 4, kPV = 4;
constexpr int kStages = 2;
constexpr int kMinBlocks = 3;
constexpr int kAttnThreads = (kQK + kPV + 1) * 32;
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
  long long ws_elems;   // FP32 elements of the workspace (debug-build checks)
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

// PK (R <= 4): the PV B fragment packs P_hi of the (at most four) query rows into columns
// 0-3 and the residual r into columns 4-7, so each V fragment meets two FP16 MMAs instead
// of four; the two column halves of the accumulator are added when the partial is written.
template <int D, bool PK>
__global__ void __launch_bounds__(kAttnThreads, kMinBlocks) heal_attn_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                       const __grid_constant__ CUtensorMap tmV,
                                                                       const AttnArgs a) {
  constexpr int kBoxes = D / 64;                    // 64-dim (128-byte) boxes per row
  constexpr int kTileBytes = kBlk * D * 2;          // one of K / V
  constexpr int kStageBytes = 2 * kTileBytes;
  constexpr int kKSteps32 = D / 32;                 // k32 steps of the integer MMA
  constexpr int kDT = D / 16 / kPV;                 // 16-dim blocks of O per PV warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;                                                  // kStages x kStageBytes
  uint4* pb = reinterpret_cast<uint4*>(smem + kStages * kStageBytes);      // [2][kQK steps][32 lanes]
  uint4* qf_sm = pb + 2 * kQK * 32;                                        // [kKSteps32][32 lanes]
  float* sc_sm = reinterpret_cast<float*>(qf_sm + kKSteps32 * 32);         // [kStages][K, V][kBlk]
  float* meta = sc_sm + kStages * 2 * kBlk;                                // [2][16]: scale of O per row, E
  float* red = meta + 2 * 16;                                              // [2][kQK][kRows] block maxima
  float* lsum = red + 2 * kQK * kRows;                                     // [kQK][kRows] row sums
  float* mq = lsum + kQK * kRows;                                          // [kRows] row maxima
  uint64_t* full = reinterpret_cast<uint64_t*>(mq + kRows);                // [S] K tile, [S] V tile + scales
  uint64_t* empty = full + 2 * kStages;                                    // [S] K released, [S] V released
  uint64_t* pready = empty + 2 * kStages;                                  // [2] P' written (QK -> PV)
  uint64_t* pfree = pready + 2;                                            // [2] P' consumed (PV -> QK)
  uint64_t* mxbar = pfree + 2;                                             // [2] block maxima exchanged
  uint64_t* finbar = mxbar + 2;                                            // row sums exchanged
  uint64_t* qfbar = finbar + 1;                                            // Q table built
  volatile int* abort_flag = reinterpret_cast<volatile int*>(qfbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long u0 = unit_begin(a.total, a.grid, c), u1 = unit_begin(a.total, a.grid, c + 1);
  pdl_launch_dependents();   // the combine kernel may be scheduled; it waits for us
  pdl_wait_prerequisites();  // Q, the caches and kv_len may come from the preceding kernel

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&full[kStages + s], 1);
      mbar_init(&empty[s], kQK);
      mbar_init(&empty[kStages + s], kPV);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pready[b], kQK);
      mbar_init(&pfree[b], kPV);
      mbar_init(&mxbar[b], kQK);
    }
    mbar_init(finbar, kQK);
    mbar_init(qfbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kQK + kPV) {
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
        // K half: refilled as soon as the QK warps finish QK^T on the previous tile
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

  const int R = a.R;
  const int g8 = lane >> 2;                   // token row (S^T) / dim row (O^T) / query of B fragments
  const int qc = 2 * (lane & 3);              // this lane's query rows qc, qc + 1
  bool ok = true;

  if (warp < kQK) {
    // ================================ QK warps ================================
    // Fragment layouts (mma.sync, g8 = lane / 4, c = lane % 4): S^T = K Q^T with
    // m16n8k32 integer MMAs, rows = this warp's 16 tokens, columns = the 8 query rows; the
    // C fragment of this lane holds tokens g8, g8 + 8 of query rows qc, qc + 1.  Byte
    // order in the K dimension: slot 4c + j of a 16-slot half holds dim
    // {2c, 2c + 1, 2c + 8, 2c + 9}[j]; both operands use it (a dot product does not
    // depend on the order of its terms).
    const int w = warp;
    const int tw = w * 16;                    // this warp's first token inside the tile
    float sqc[2] = {0.0f, 0.0f};             // fp32(fp32(s_q * softmax_scale) * log2(e)) per row
    int pos[2] = {0, 0};
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
    int E_run = 0;                            // power of two folded into P (decreases only)
    bool have_E = false;
    int cur_p = -1, b = 0, hkv = 0, klen = 0;
    int j = 0, nfin = 0, nsetup = 0;

    auto finalize = [&](int p) {
      // row sums over this warp's lanes, then over the four QK warps in order
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = l_run[e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (g8 == 0) {
          lsum[w * kRows + qc + e] = l;
          if (w == 0) mq[qc + e] = m_run[e];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(finbar);
      if (!mbar_wait(finbar, (uint32_t)(nfin & 1), abort_flag, a.status, 215)) ok = false;
      ++nfin;
      if (ok && w == 0 && lane < R) {
        float L = 0.0f;
        for (int ww = 0; ww < kQK; ++ww) L = __fadd_rn(L, lsum[ww * kRows + lane]);
        float* sl = slot_ptr(a.ws, c, p, R, D) + R * D;
        if (HEAL_DCHECK((long long)(sl + 2 * lane + 1 - a.ws) < a.ws_elems, a.status, 250)) {
          sl[2 * lane] = mq[lane];
          sl[2 * lane + 1] = L;
        }
      }
    };

    for (long long u = u0; u < u1 && ok; ++u) {
      const int p = (int)(u / a.nblk), blk = (int)(u % a.nblk);
      if (p != cur_p) {
        if (cur_p >= 0) {
          finalize(cur_p);
          if (!ok) break;
        }
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
          sqc[e] = real ? __fmul_rn(__fmul_rn(__ldg(a.qs + ((long long)(b * a.Hq + hkv * a.G + gq) * a.Tq + tq)),
                                              a.scale), kLog2e)
                        : 0.0f;
          pos[e] = klen - a.Tq + tq;
        }
        // B fragments of Q^T (query row g8), byte-split, one table per CTA:
        // entry [s][lane] = (hi slots 0-15, hi slots 16-31, lo slots 0-15, lo slots 16-31).
        // Warp 0 rebuilds it once every QK warp is past the previous pair (finalize).
        if (w == 0) {
          const int r = g8;
          const bool real = r < R;
          const int tq = real ? r / a.G : 0, gq = real ? r % a.G : 0;
          const long long qrow = ((long long)(b * a.Hq + hkv * a.G + gq) * a.Tq + tq);
#pragma unroll
          for (int s32 = 0; s32 < kKSteps32; ++s32) {
            uint32_t wq[4] = {0u, 0u, 0u, 0u};
            if (real) {
              const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.q + qrow * D + s32 * 32 + qc);
#pragma unroll
              for (int i = 0; i < 4; ++i) wq[i] = __ldg(qp + 4 * i);   // dims 32s + 8i + 2c, +1
            }
            qf_sm[s32 * 32 + lane] = make_uint4(hi_bytes(wq[0], wq[1]), hi_bytes(wq[2], wq[3]),
                                                lo_bytes(wq[0], wq[1]), lo_bytes(wq[2], wq[3]));
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(qfbar);
        }
        if (!mbar_wait(qfbar, (uint32_t)(nsetup & 1), abort_flag, a.status, 216)) {
          ok = false;
          break;
        }
        ++nsetup;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          m_run[e] = -INFINITY;
          l_run[e] = 0.0f;
        }
        E_run = 0;
        have_E = false;
      }
      const int t0 = blk * kBlk;
      if (t0 >= klen) continue;
      const int s = j % kStages;
      const uint32_t ph = (uint32_t)(j / kStages) & 1u;
      const int jb = j & 1;
      const uint32_t jph = (uint32_t)(j >> 1) & 1u;
      ++j;
      if (!mbar_wait(&full[s], ph, abort_flag, a.status, 210)) {
        ok = false;
        break;
      }
      const uint32_t kst = smem_u32(stages + s * kStageBytes);
      const float* sks = sc_sm + (s * 2 + 0) * kBlk;   // K scales of this block's 64 tokens
      const float* svs = sc_sm + (s * 2 + 1) * kBlk;   // V scales

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
      // every ldmatrix of the K tile has been consumed and the K scales this lane needs
      // are in registers: release the K half before the logit arithmetic
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
          // S = 65536*S_hh + low, low = 256*S_x + S_ll (|low| < 2^31 for head_dim <= 128)
          const int low = (sxa[i] + sxb[i]) * 256 + sll[i];
          const bool real = r < R;
          const bool vis = real && t < klen && (!a.causal || t <= pos[e]);
          float xv;
          if (!real) {
            xv = 0.0f;                          // padding query row: finite, never written
          } else if (!vis) {
            xv = -INFINITY;
          } else {
            const float sf = __fmaf_rn(small_int_to_float(shh[i]), 65536.0f, __int2float_rn(low));
            xv = __fmul_rn(__fmul_rn(sf, skr[th]), sqc[e]);
            if (a.qk_out) {
              const long long S = (long long)shh[i] * 65536LL + (long long)low;
              const int tq = r / a.G, gq = r % a.G;
              const long long qi = ((long long)(b * a.Hq + hkv * a.G + gq) * a.Tq + tq) * a.Tmax + t;
              if (HEAL_DCHECK(qi < (long long)a.B * a.Hq * a.Tq * a.Tmax && t < a.Tmax, a.status, 251))
                a.qk_out[qi] = S;
            }
          }
          x[th][e] = xv;
        }
      }

      // ---- the block's maximum per query row, shared by the four QK warps ----
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float bm = fmaxf(x[0][e], x[1][e]);
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
        if (g8 == 0) red[(jb * kQK + w) * kRows + qc + e] = bm;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&mxbar[jb]);
      // the V tile's scales arrive with it: wait for the stage without consuming it
      if (!mbar_wait(&mxbar[jb], jph, abort_flag, a.status, 212) ||
          !mbar_wait(&full[kStages + s], ph, abort_flag, a.status, 211)) {
        ok = false;
        break;
      }
      float alpha[2], pv[2][2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float bm = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kQK; ++ww) bm = fmaxf(bm, red[(jb * kQK + ww) * kRows + qc + e]);
        const float m_new = fmaxf(m_run[e], bm);
        if (m_new == -INFINITY) {
          alpha[e] = 1.0f;
          pv[0][e] = pv[1][e] = 0.0f;
        } else {
          alpha[e] = (m_run[e] == -INFINITY) ? 0.0f : fast_exp2(m_run[e] - m_new);
#pragma unroll
          for (int th = 0; th < 2; ++th) pv[th][e] = (x[th][e] == -INFINITY) ? 0.0f : fast_exp2(x[th][e] - m_new);
        }
        l_run[e] = __fadd_rn(__fmul_rn(l_run[e], alpha[e]), __fadd_rn(pv[0][e], pv[1][e]));
        m_run[e] = m_new;
      }
      // power of two for this block: the largest visible V scale times 2^E in [32, 64)
      // (V scales are non-negative, so their bit patterns order like the floats)
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

      // ---- P' = P * s_v * 2^E (S^T layout), moved to the B layout of PV: lane (g8, c)
      // needs tokens 2c, 2c + 1, 2c + 8, 2c + 9 of query row g8 (PK: of row g8 & 3).  Token
      // 2c + jj lives in lane 4 * (2c + jj) + row / 2 (halves th = 0 / 1 for +0 / +8), the row
      // in slot row & 1.
      float pp[2][2];
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const int t = t0 + tw + th * 8 + g8;
        const float svt = mul_pow2(svs[t - t0], E_run);   // s_v * 2^E, in [0, 64)
#pragma unroll
        for (int e = 0; e < 2; ++e) pp[th][e] = __fmul_rn(pv[th][e], (pv[th][e] != 0.0f) ? svt : 0.0f);
      }
      float pt[2][2];                            // [token half][jj]: P' of token 8*half + 2c + jj, query g8
      {
        const int cq = lane & 3;
        const bool odd = (g8 & 1) != 0;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int src = 4 * (2 * cq + jj) + ((PK ? (g8 & 3) : g8) >> 1);
#pragma unroll
          for (int th = 0; th < 2; ++th) {
            const float v0 = __shfl_sync(0xffffffffu, pp[th][0], src);
            const float v1 = __shfl_sync(0xffffffffu, pp[th][1], src);
            pt[th][jj] = odd ? v1 : v0;
          }
        }
      }
      // FP16 P_hi and residual r = P' - P_hi: the B fragments of PV (the PV warps form the
      // 256x copies themselves).  PK: columns 4-7 (g8 >= 4) carry r, so both slots hold
      // the column's own part.
      uint32_t ph_[2], pr_[2];
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const __half2 h = __floats2half2_rn(pt[th][0], pt[th][1]);
        const float2 hf = __half22float2(h);
        const __half2 rr = __floats2half2_rn(__fsub_rn(pt[th][0], hf.x), __fsub_rn(pt[th][1], hf.y));
        ph_[th] = *reinterpret_cast<const uint32_t*>(&h);
        pr_[th] = *reinterpret_cast<const uint32_t*>(&rr);
        if (PK && g8 >= 4) ph_[th] = pr_[th];
      }
      // hand the block to the PV warps (the buffer is free once they finished block j - 2)
      if (!mbar_wait(&pfree[jb], jph ^ 1u, abort_flag, a.status, 213)) {
        ok = false;
        break;
      }
      pb[(jb * kQK + w) * 32 + lane] = make_uint4(ph_[0], ph_[1], pr_[0], pr_[1]);
      if (w == 0) {
        if (g8 == 0) {
          meta[jb * 16 + qc] = __fmul_rn(alpha[0], escale);
          meta[jb * 16 + qc + 1] = __fmul_rn(alpha[1], escale);
        }
        if (lane == 0) meta[jb * 16 + 8] = __int_as_float(E_run);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[jb]);
    }
    if (ok && cur_p >= 0) finalize(cur_p);
    return;
  }

  // ================================ PV warps ================================
  // O^T = V^T P'^T with m16n8k16 FP16 MMAs: rows = 16 dims, columns = the 8 query rows;
  // this warp owns dims [v * D/4, (v + 1) * D/4) of every row over all 64 tokens.
  const int v = warp - kQK;
  float om[kDT][4];                           // O^T accumulator (units of 2^E_run)
#pragma unroll
  for (int dl = 0; dl < kDT; ++dl)
#pragma unroll
    for (int e = 0; e < 4; ++e) om[dl][e] = 0.0f;
  int E_run = 0;
  int cur_p = -1, klen = 0;
  int j = 0;

  auto finalize_o = [&](int p) {
    float* sl = slot_ptr(a.ws, c, p, R, D);
    if constexpr (PK) {
      // columns 4-7 (lanes with c >= 2) hold the residual part of rows 0-3
#pragma unroll
      for (int dl = 0; dl < kDT; ++dl)
#pragma unroll
        for (int e = 0; e < 4; ++e) om[dl][e] = __fadd_rn(om[dl][e], __shfl_xor_sync(0xffffffffu, om[dl][e], 2));
    }
#pragma unroll
    for (int dl = 0; dl < kDT; ++dl)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = (v * kDT + dl) * 16 + g8 + ((e >> 1) << 3);
        const int r = qc + (e & 1);
        if (r < R && (!PK || qc < 4) && HEAL_DCHECK((long long)(sl + r * D + d - a.ws) < a.ws_elems, a.status, 252))
          sl[r * D + d] = mul_pow2(om[dl][e], -E_run);   // true units (x 2^-E_run)
        om[dl][e] = 0.0f;
      }
  };

  for (long long u = u0; u < u1 && ok; ++u) {
    const int p = (int)(u / a.nblk), blk = (int)(u % a.nblk);
    if (p != cur_p) {
      if (cur_p >= 0) finalize_o(cur_p);
      cur_p = p;
      klen = __ldg(a.kv_len + p / a.Hkv);
      E_run = 0;
    }
    const int t0 = blk * kBlk;
    if (t0 >= klen) continue;
    const int s = j % kStages;
    const uint32_t ph = (uint32_t)(j / kStages) & 1u;
    const int jb = j & 1;
    const uint32_t jph = (uint32_t)(j >> 1) & 1u;
    ++j;
    if (!mbar_wait(&pready[jb], jph, abort_flag, a.status, 220) ||
        !mbar_wait(&full[kStages + s], ph, abort_flag, a.status, 221)) {
      ok = false;
      break;
    }
    const uint32_t vst = smem_u32(stages + s * kStageBytes) + kTileBytes;
    // rescale O^T columns qc, qc + 1 by the block's softmax step and change of 2^E
    const int qr = PK ? (qc & 3) : qc;                 // the query rows of this lane's columns
    const float a0 = meta[jb * 16 + qr], a1 = meta[jb * 16 + qr + 1];
    E_run = __float_as_int(meta[jb * 16 + 8]);
    if (!__all_sync(0xffffffffu, a0 == 1.0f && a1 == 1.0f)) {
#pragma unroll
      for (int dl = 0; dl < kDT; ++dl) {
        om[dl][0] = __fmul_rn(om[dl][0], a0);
        om[dl][1] = __fmul_rn(om[dl][1], a1);
        om[dl][2] = __fmul_rn(om[dl][2], a0);
        om[dl][3] = __fmul_rn(om[dl][3], a1);
      }
    }
    // ---- O^T += V^T P'^T  (256*hi*P + lo*P with P = P_hi + r), 16 tokens per step ----
#pragma unroll
    for (int ts = 0; ts < kQK; ++ts) {
      const uint4 f = pb[(jb * kQK + ts) * 32 + lane];               // P_hi, r
      // 256 * P_hi and 256 * r: exact (powers of two; |P'| < 64)
      const __half2 k256 = __half2half2(__ushort_as_half(0x5C00));
      uint4 fh, fr;                                                  // (256 x, x) of P_hi / r
      if constexpr (PK) {
        const __half2 h0 = __hmul2(*reinterpret_cast<const __half2*>(&f.x), k256);
        const __half2 h1 = __hmul2(*reinterpret_cast<const __half2*>(&f.y), k256);
        fh = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1), f.x, f.y);
        fr = fh;
      } else {
        const __half2 h0 = __hmul2(*reinterpret_cast<const __half2*>(&f.x), k256);
        const __half2 h1 = __hmul2(*reinterpret_cast<const __half2*>(&f.y), k256);
        const __half2 r0 = __hmul2(*reinterpret_cast<const __half2*>(&f.z), k256);
        const __half2 r1 = __hmul2(*reinterpret_cast<const __half2*>(&f.w), k256);
        fh = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1), f.x, f.y);
        fr = make_uint4(*reinterpret_cast<const uint32_t*>(&r0), *reinterpret_cast<const uint32_t*>(&r1), f.z, f.w);
      }
#pragma unroll
      for (int dl = 0; dl < kDT; ++dl) {
        const int dt = v * kDT + dl;
        const int mi = lane >> 3;
        const int trow = ts * 16 + ((mi >> 1) << 3) + (lane & 7);
        const int ch = 2 * dt + (mi & 1);
        const uint32_t addr = vst + (ch >> 3) * 8192 + trow * 128 + ((((ch & 7) ^ (trow & 7))) << 4);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(addr, r0, r1, r2, r3);
        const uint32_t h0 = hi_pair(r0), h1 = hi_pair(r1), h2 = hi_pair(r2), h3 = hi_pair(r3);
        const uint32_t l0 = lo_pair(r0), l1 = lo_pair(r1), l2 = lo_pair(r2), l3 = lo_pair(r3);
        mma16816(om[dl], h0, h1, h2, h3, fh.x, fh.y);
        mma16816(om[dl], l0, l1, l2, l3, fh.z, fh.w);
        if constexpr (!PK) {
          mma16816(om[dl], h0, h1, h2, h3, fr.x, fr.y);
          mma16816(om[dl], l0, l1, l2, l3, fr.z, fr.w);
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[kStages + s]);   // V tile consumed
      mbar_arrive(&pfree[jb]);            // P' buffer consumed
    }
  }
  if (ok && cur_p >= 0) finalize_o(cur_p);
}

// out[b, hq, tq, :] = sum_c o_c 2^(m_c - M) / sum_c l_c 2^(m_c - M), c ascending.
// When a pair's partials come from at most kCombBatch CTAs (the usual case) m, l and o are
// requested together, so the whole merge costs one memory round trip; otherwise the
// partials of kCombBatch CTAs are requested together per step, the maximum first.  Either
// way they are applied one by one in ascending CTA order, so the sums are the same as a
// one-at-a-time loop.
constexpr int kCombBatch = 8;
template <int D>
__global__ void __launch_bounds__(D) heal_attn_combine_kernel(const AttnArgs a) {
  pdl_launch_dependents();              // the next kernel may be scheduled; it waits for this grid
  pdl_wait_prerequisites();             // the decode kernel that wrote the partials has completed
  const int pr = blockIdx.x;            // (pair, row)
  const int p = pr / a.R, r = pr % a.R;
  const int d = threadIdx.x;
  const long long ufirst = (long long)p * a.nblk, ulast = ufirst + a.nblk - 1;
  const int c0 = cta_of(ufirst, a.total, a.grid), c1 = cta_of(ulast, a.total, a.grid);
  float M = -INFINITY, L = 0.0f, O = 0.0f;
  auto apply = [&](const float (&m)[kCombBatch], const float (&l)[kCombBatch], const float (&o)[kCombBatch]) {
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) {
      if (m[t] == -INFINITY) continue;
      const float f = exp2f(m[t] - M);
      L = __fadd_rn(L, __fmul_rn(l[t], f));
      O = __fadd_rn(O, __fmul_rn(o[t], f));
    }
  };
  auto load = [&](int cb, float (&m)[kCombBatch], float (&l)[kCombBatch], float (&o)[kCombBatch]) {
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) {
      const bool in = cb + t <= c1;
      const float* sl = slot_ptr(a.ws, in ? cb + t : c0, p, a.R, D);
      m[t] = in ? sl[a.R * D + 2 * r] : -INFINITY;
      l[t] = in ? sl[a.R * D + 2 * r + 1] : 0.0f;
      o[t] = in ? sl[r * D + d] : 0.0f;
    }
    // all of them in flight before any is used (not sunk into the adds that need them)
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) asm volatile("" ::"f"(m[t]), "f"(l[t]), "f"(o[t]));
  };
  if (c1 - c0 < kCombBatch) {
    float m[kCombBatch], l[kCombBatch], o[kCombBatch];
    load(c0, m, l, o);
#pragma unroll
    for (int t = 0; t < kCombBatch; ++t) M = fmaxf(M, m[t]);
    apply(m, l, o);
  } else {
    for (int cb = c0; cb <= c1; cb += kCombBatch) {
      float m[kCombBatch];
#pragma unroll
      for (int t = 0; t < kCombBatch; ++t)
        m[t] = (cb + t <= c1) ? slot_ptr(a.ws, cb + t, p, a.R, D)[a.R * D + 2 * r] : -INFINITY;
#pragma unroll
      for (int t = 0; t < kCombBatch; ++t) M = fmaxf(M, m[t]);
    }
    for (int cb = c0; cb <= c1; cb += kCombBatch) {
      float m[kCombBatch], l[kCombBatch], o[kCombBatch];
      load(cb, m, l, o);
      apply(m, l, o);
    }
  }
  const int b = p / a.Hkv, hkv = p % a.Hkv;
  const int tq = r / a.G, g = r % a.G;
  // a query with no visible token (causal, kv_len < Tq) gets zeros
  const long long oi = (((long long)(b * a.Hq + hkv * a.G + g) * a.Tq + tq) * D) + d;
  if (HEAL_DCHECK(oi < (long long)a.B * a.Hq * a.Tq * D, a.status, 253)) a.out[oi] = L > 0.0f ? __fdiv_rn(O, L) : 0.0f;
}

template <int D>
constexpr int attn_smem_bytes() {
  return kStages * (2 * kBlk * D * 2)          // K / V stages
         + 2 * kQK * 32 * 16                   // P' operand buffers
         + (D / 32) * 32 * 16                  // Q table
         + kStages * 2 * kBlk * 4              // K / V scales
         + (2 * 16 + 2 * kQK * kRows + kQK * kRows + kRows) * 4   // meta, maxima, sums
         + (4 * kStages + 8) * 8 + 16          // barriers, abort flag
         + 1024;                               // alignment
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
    if (cudaFuncSetAttribute(heal_attn_decode_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem_bytes<128>()) != cudaSuccess ||
        cudaFuncSetAttribute(heal_attn_decode_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem_bytes<128>()) != cudaSuccess ||
        cudaFuncSetAttribute(heal_attn_decode_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem_bytes<64>()) != cudaSuccess ||
        cudaFuncSetAttribute(heal_attn_decode_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem_bytes<64>()) != cudaSuccess)
      return HEAL_ERR_CUDA;
    // both forms of a head size are built for the same residency (launch bounds)
    int p0 = 0, p1 = 0;
    if (D == 128) {
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p0, heal_attn_decode_kernel<128, false>, kAttnThreads,
                                                    attn_smem_bytes<128>());
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p1, heal_attn_decode_kernel<128, true>, kAttnThreads,
                                                    attn_smem_bytes<128>());
    } else {
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p0, heal_attn_decode_kernel<64, false>, kAttnThreads,
                                                    attn_smem_bytes<64>());
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p1, heal_attn_decode_kernel<64, true>, kAttnThreads,
                                                    attn_smem_bytes<64>());
    }
    per_sm = p0 < p1 ? p0 : p1;
    if (per_sm < 1) per_sm = 1;
    per_sm_cache[dev][di] = per_sm;
  }
  long long grid = (long long)sms * per_sm;
  if (grid > kMaxGrid) grid = kMaxGrid;
  if (grid > a.total) grid = a.total;
  a.grid = (int)grid;
  a.status = device_status_ptr();
  a.ws_elems = (long long)(ws_bytes / sizeof(float));
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
  const bool pk = R <= 4;
  const dim3 g(a.grid), t(kAttnThreads);
  if (D == 128) {
    e = pk ? launch_pdl(heal_attn_decode_kernel<128, true>, g, t, (size_t)attn_smem_bytes<128>(), stream, tk, tv, a)
           : launch_pdl(heal_attn_decode_kernel<128, false>, g, t, (size_t)attn_smem_bytes<128>(), stream, tk, tv, a);
    if (e == cudaSuccess) e = launch_pdl(heal_attn_combine_kernel<128>, dim3(B * Hkv * R), dim3(128), 0, stream, a);
  } else {
    e = pk ? launch_pdl(heal_attn_decode_kernel<64, true>, g, t, (size_t)attn_smem_bytes<64>(), stream, tk, tv, a)
           : launch_pdl(heal_attn_decode_kernel<64, false>, g, t, (size_t)attn_smem_bytes<64>(), stream, tk, tv, a);
    if (e == cudaSuccess) e = launch_pdl(heal_attn_combine_kernel<64>, dim3(B * Hkv * R), dim3(64), 0, stream, a);
  }
  if (e != cudaSuccess) return HEAL_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

}  // namespace heal
