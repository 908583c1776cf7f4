// attention_prefill.cu -- K5 for many query rows per KV head (prefill / chunked prefill):
// INT16 attention on the tcgen05 tensor cores (gist.science technical summary, section
// 2.A, "Mechanism": the INT16 tensor is unpacked into two 16-bit tensors for the attention
// contractions).
//
// Arithmetic (the same definition as the decode kernel):
//   q = 256*hi + lo, hi = q >> 8 (s8), lo = q & 255 (u8);
//   S_int = 65536*S_hh + 256*S_x + S_ll, S_hh = Qhi.Khi, S_x = Qhi.Klo + Qlo.Khi, S_ll = Qlo.Klo,
// four tcgen05.mma.kind::i8 products per 32-wide slice of the head dimension, each exact in
// its 32-bit TMEM accumulator (for head_dim 128 no partial sum reaches 2^24), combined in
// int64 by the softmax threads.
//   logit * log2(e) = fp32(fp32(S_int) * s_k) * (s_q * scale * log2 e), the last factor
// applied inside the exponent's FMA; fp32(S_int) is 65536*S_hh + fp32(256*S_x + S_ll)
// rounded once more (the decode kernel forms the logit through FP64; the two agree to a
// few units in the last place).  Online softmax in base 2 with a lazy maximum: the
// reference maximum of a row moves only when a block's maximum exceeds it by more than 8,
// so P <= 2^8 and the running O is rescaled only on those blocks.
//   P' = P * s_v * 2^E, E per (batch, kv head) such that max s_v * 2^E lies in [32, 64);
//   P' = P_hi + r with P_hi = fp16(P'), r = fp16(P' - P_hi);
//   O += P_hi.(256 V_hi) + P_hi.V_lo + r.(256 V_hi) + r.V_lo     (four kind::f16 MMAs)
// where 256*V_hi and V_lo are exact FP16 values, so the sum over the two V parts is
// P'_t * v_t up to the FP32 accumulation.  tcgen05's FP32 accumulation truncates, so each
// 64-token block's PV product starts a fresh TMEM accumulator and the softmax threads add
// the block results in FP32 round-to-nearest, in ascending block order, into O held in
// registers.  O_out = O * 2^-E / l.
//
// Two launches.  A conversion pass writes the byte planes (Khi/Klo s8/u8, 256*Vhi/Vlo FP16,
// Qhi/Qlo) into the workspace in the layouts the MMAs read, and the per-(batch, kv head)
// exponent E; it reads each cache element once.  The attention kernel then streams only
// MMA-ready tiles by TMA.
//
// Attention kernel, one CTA per (batch, query head, 128-row query tile), the tiles with
// the most key blocks first, 10 warps:
//   warp 0   TMA producer: Q planes once; per 64-token key block the K planes, the V
//            planes and the block's K/V scales, each in its own ring
//   warp 1   MMA issuer (one thread): QK(j+1) is issued before PV(j), so the tensor pipe
//            works on the next block's scores while the softmax threads build P(j)
//   warps 2-9 softmax: thread (warp, lane) owns query row 32*(warp%4) + lane (its TMEM
//            lane) and half (warp-2)/4 of each block's 64 tokens and of O's 128 columns
// TMEM (512 columns): two S buffers of three 64-column int32 accumulators, the block's PV
// product in the last 128 columns.  Every wait is a bounded mbarrier wait.
#include <cuda_fp16.h>

#include <cmath>
#include <type_traits>

#include "heal_internal.h"
#include "heal_ptx.cuh"

namespace heal {

namespace {

constexpr int kPD = 128;            // head dim (the prefill path is built for 128)
constexpr int kPM = 128;            // query rows per CTA
constexpr int kPN = 64;             // tokens per key block
constexpr int kKSt = 2;             // K plane stages
constexpr int kVSt = 2;             // V plane stages
constexpr int kScSt = 4;            // scale stages
#ifndef HEAL_PREFILL_SM_WARPS
#define HEAL_PREFILL_SM_WARPS 8
#endif
constexpr int kSmWarps = HEAL_PREFILL_SM_WARPS;   // softmax warps: 8 or 16
constexpr int kGroups = kSmWarps / 4;             // warps sharing one TMEM lane quarter
constexpr int kTokPer = kPN / kGroups;            // tokens of a block per softmax thread
constexpr int kOCols = kPD / kGroups;             // columns of O per softmax thread
static_assert(kSmWarps == 8 || kSmWarps == 16, "8 or 16 softmax warps");
constexpr int kPThreads = (2 + kSmWarps) * 32;
constexpr int kSmWarp0 = 2;         // first softmax warp
constexpr float kLog2eP = 1.4426950408889634f;

// shared-memory layout (bytes from a 1024-aligned base)
constexpr int kOffQhi = 0;
constexpr int kOffQlo = kOffQhi + kPM * kPD;                 // 16 KB planes
constexpr int kOffK = kOffQlo + kPM * kPD;                   // per stage: Khi 8 KB, Klo 8 KB
constexpr int kKStage = 2 * kPN * kPD;
constexpr int kOffV = kOffK + kKSt * kKStage;                // per stage: Vh 16 KB, Vl 16 KB
constexpr int kVStage = 2 * kPN * kPD * 2;
constexpr int kOffP = kOffV + kVSt * kVStage;                // per buffer: Phi 16 KB, Pr 16 KB
constexpr int kPBuf = 2 * kPM * kPN * 2;
constexpr int kOffSc = kOffP + 2 * kPBuf;                    // per stage: 64 K scales, 64 V scales
constexpr int kScStage = 2 * kPN * 4;
constexpr int kOffRed = kOffSc + kScSt * kScStage;           // [2 buffers][kGroups][128] block maxima
constexpr int kOffL = kOffRed + 2 * kGroups * kPM * 4;       // [kGroups][128] row sums
constexpr int kOffBar = kOffL + kGroups * kPM * 4;
// barriers: qfull, kfull[kKSt], kfree[kKSt], vfull[kVSt], vfree[kVSt], scfull[kScSt],
// scfree[kScSt], sfull[2], sfree[2], pready[2], pfree[2], odone, drain, mx[2][4] (block
// maxima exchanged by the two warps of a lane quarter), fin[4] (their row sums), ofree
constexpr int kNumBars = 1 + 2 * kKSt + 2 * kVSt + 2 * kScSt + 8 + 2 + 8 + 4 + 1;
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmem + 8;
constexpr int kPSmem = kOffAbort + 8 + 1024;                 // + alignment slack

struct PrefillArgs {
  const float* qs;        // [B, Hq, Tq]
  const float* ks;        // [B, Hkv, Tmax]
  const float* vs;        // [B, Hkv, Tmax]
  const int32_t* kv_len;  // [B]
  const int* E;           // [B, Hkv] (conversion pass output)
  const float* cv;        // [B, Hkv, Tmax] s_v * 2^E, 0 past kv_len (conversion pass output)
  long long* qk_out;      // nullable [B, Hq, Tq, Tmax]
  float* out;             // [B, Hq, Tq, 128]
  int B, Hq, Hkv, G, Tq, Tmax, nqt, causal;
  float scale;
  unsigned int* status;
};

struct PlanesArgs {
  const int16_t* q;       // [B, Hq, Tq, 128]
  const int16_t* k;       // [B, Hkv, Tmax, 128]
  const int16_t* v;
  const float* vs;        // [B, Hkv, Tmax]
  const int32_t* kv_len;
  uint8_t* khi;           // [B*Hkv*Tmax, 128] s8
  uint8_t* klo;           //                   u8
  __half* vh;             // [B*Hkv*Tmax, 128] 256*hi
  __half* vl;             //                   lo
  uint8_t* qhi;           // [B*Hq*Tq, 128]
  uint8_t* qlo;
  int* E;                 // [B, Hkv]
  float* cv;              // [B, Hkv, Tmax]
  long long nk8;          // K/V elements / 8
  long long nq8;          // Q elements / 8
  int B, Hkv, Tmax;
  const uint8_t* ws;      // workspace base and size (debug-build checks of the plane writes)
  long long ws_bytes;
  unsigned int* status;
};

// debug builds: the byte range [p, p + n) lies inside the workspace
__device__ __forceinline__ bool in_ws(const PlanesArgs& a, const void* p, long long n, int site) {
#ifdef HEAL_DEBUG
  const long long off = (long long)(reinterpret_cast<const uint8_t*>(p) - a.ws);
  return debug_check(off >= 0 && off + n <= a.ws_bytes, a.status, site);
#else
  (void)a, (void)p, (void)n, (void)site;
  return true;
#endif
}

// x * 2^e exactly for |e| <= 252 (two steps, each a normal power of two).
__device__ __forceinline__ float mul_pow2_p(float x, int e) {
  const int e1 = e / 2, e2 = e - e1;
  return __fmul_rn(__fmul_rn(x, __int_as_float((127 + e1) << 23)), __int_as_float((127 + e2) << 23));
}

// Eight int16 values (a uint4) -> their high bytes and low bytes (two uint2).
__device__ __forceinline__ void bytes8(const uint4 w, uint2& hi, uint2& lo) {
  hi.x = __byte_perm(w.x, w.y, 0x7531);
  hi.y = __byte_perm(w.z, w.w, 0x7531);
  lo.x = __byte_perm(w.x, w.y, 0x6420);
  lo.y = __byte_perm(w.z, w.w, 0x6420);
}

// Two int16 values packed in x -> FP16 (256*hi0, 256*hi1) and (lo0, lo1), both exact.
__device__ __forceinline__ void vparts2(uint32_t x, uint32_t& h, uint32_t& l) {
  const int v0 = (int)(short)(x & 0xFFFFu), v1 = (int)(short)(x >> 16);
  const __half2 hh = __floats2half2_rn((float)((v0 >> 8) * 256), (float)((v1 >> 8) * 256));
  const __half2 ll = __floats2half2_rn((float)(v0 & 255), (float)(v1 & 255));
  h = *reinterpret_cast<const uint32_t*>(&hh);
  l = *reinterpret_cast<const uint32_t*>(&ll);
}

// Conversion pass.  blockIdx.y: 0 K planes, 1 V planes, 2 Q planes, 3 the exponent E of
// one (batch, kv head) per block.  Pure streaming; grid-stride over 16-byte chunks.
__global__ void __launch_bounds__(256) heal_attn_planes_kernel(const PlanesArgs a) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  if (blockIdx.y == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(a.k);
    uint2* dh = reinterpret_cast<uint2*>(a.khi);
    uint2* dl = reinterpret_cast<uint2*>(a.klo);
    for (long long i = tid; i < a.nk8; i += stride) {
      uint2 h, l;
      bytes8(__ldg(src + i), h, l);
      if (in_ws(a, dh + i, 8, 270) && in_ws(a, dl + i, 8, 271)) {
        dh[i] = h;
        dl[i] = l;
      }
    }
  } else if (blockIdx.y == 1) {
    const uint4* src = reinterpret_cast<const uint4*>(a.v);
    uint4* dh = reinterpret_cast<uint4*>(a.vh);
    uint4* dl = reinterpret_cast<uint4*>(a.vl);
    for (long long i = tid; i < a.nk8; i += stride) {
      const uint4 w = __ldg(src + i);
      uint4 h, l;
      vparts2(w.x, h.x, l.x);
      vparts2(w.y, h.y, l.y);
      vparts2(w.z, h.z, l.z);
      vparts2(w.w, h.w, l.w);
      if (in_ws(a, dh + i, 16, 272) && in_ws(a, dl + i, 16, 273)) {
        dh[i] = h;
        dl[i] = l;
      }
    }
  } else if (blockIdx.y == 2) {
    const uint4* src = reinterpret_cast<const uint4*>(a.q);
    uint2* dh = reinterpret_cast<uint2*>(a.qhi);
    uint2* dl = reinterpret_cast<uint2*>(a.qlo);
    for (long long i = tid; i < a.nq8; i += stride) {
      uint2 h, l;
      bytes8(__ldg(src + i), h, l);
      if (in_ws(a, dh + i, 8, 274) && in_ws(a, dl + i, 8, 275)) {
        dh[i] = h;
        dl[i] = l;
      }
    }
  } else {
    // E of (b, hkv) = blockIdx.x: the largest V scale of the visible tokens times 2^E in
    // [32, 64).  V scales are non-negative, so their bit patterns order like the floats.
    // Then cv = s_v * 2^E for the visible tokens and 0 for the rest of the cache rows.
    __shared__ unsigned int wmax[8];
    __shared__ int e_sh;
    const int p = blockIdx.x;
    if (p >= a.B * a.Hkv) return;
    const int b = p / a.Hkv;
    const int klen = min(max(__ldg(a.kv_len + b), 0), a.Tmax);
    const float* s = a.vs + (long long)p * a.Tmax;
    unsigned int um = 0u;
    for (int t = threadIdx.x; t < klen; t += blockDim.x) um = max(um, __float_as_uint(__ldg(s + t)));
    um = __reduce_max_sync(0xffffffffu, um);
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = um;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned int m = 0u;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = max(m, wmax[w]);
      const float smax = __uint_as_float(m);
      e_sh = (smax > 0.0f) ? 5 - ilogbf(smax) : 0;
      if (in_ws(a, a.E + p, 4, 276)) a.E[p] = e_sh;
    }
    __syncthreads();
    const int E = e_sh;
    float* cv = a.cv + (long long)p * a.Tmax;
    for (int t = threadIdx.x; t < a.Tmax; t += blockDim.x)
      if (in_ws(a, cv + t, 4, 277)) cv[t] = t < klen ? mul_pow2_p(__ldg(s + t), E) : 0.0f;
  }
}

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return smem_desc_sw128(addr, 16, 1024); }
__device__ __forceinline__ uint64_t vdesc(uint32_t addr) { return smem_desc_sw128(addr, 8192, 1024); }

// A wait used only to drain copies and MMAs before the CTA exits: bounded, but not cut
// short by the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned int* status, int site) {
  volatile int never = 0;
  (void)mbar_wait(bar, parity, &never, status, site);
}

// HOOK: also write the exact S_int of every visible pair to qk_out (the test hook); a
// separate instantiation keeps that path out of the production kernel.
template <bool HOOK>
__global__ void __launch_bounds__(kPThreads, 1)
    heal_attn_prefill_kernel(const __grid_constant__ CUtensorMap tq_hi, const __grid_constant__ CUtensorMap tq_lo,
                             const __grid_constant__ CUtensorMap tk_hi, const __grid_constant__ CUtensorMap tk_lo,
                             const __grid_constant__ CUtensorMap tv_h, const __grid_constant__ CUtensorMap tv_l,
                             const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint64_t* qfull = bars;
  uint64_t* kfull = qfull + 1;
  uint64_t* kfree = kfull + kKSt;
  uint64_t* vfull = kfree + kKSt;
  uint64_t* vfree = vfull + kVSt;
  uint64_t* scfull = vfree + kVSt;
  uint64_t* scfree = scfull + kScSt;
  uint64_t* sfull = scfree + kScSt;
  uint64_t* sfree = sfull + 2;
  uint64_t* pready = sfree + 2;
  uint64_t* pfree = pready + 2;
  uint64_t* odone = pfree + 2;
  uint64_t* drain = odone + 1;
  uint64_t* mx = drain + 1;      // [2][4]
  uint64_t* fin = mx + 8;        // [4]
  uint64_t* ofree = fin + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbh = a.B * a.Hq;
  const int qt = a.nqt - 1 - (int)(blockIdx.x / nbh);   // most key blocks first
  const int bh = (int)(blockIdx.x % nbh);
  const int b = bh / a.Hq, h = bh % a.Hq, hkv = h / a.G;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < kKSt; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kfree[i], 1);
    }
    for (int i = 0; i < kVSt; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vfree[i], 1);
    }
    for (int i = 0; i < kScSt; ++i) {
      mbar_init(&scfull[i], 1);
      mbar_init(&scfree[i], kSmWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sfree[i], kSmWarps);
      mbar_init(&pready[i], kSmWarps);
      mbar_init(&pfree[i], 1);
    }
    mbar_init(odone, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&mx[i], kGroups);
    for (int i = 0; i < 4; ++i) mbar_init(&fin[i], kGroups);
    mbar_init(ofree, kSmWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  pdl_launch_dependents();
  pdl_wait_prerequisites();   // the planes and E are written by the conversion pass

  const int klen = min(max(__ldg(a.kv_len + b), 0), a.Tmax);
  const int row0 = qt * kPM;
  int kend = klen;
  if (a.causal) kend = min(kend, klen - a.Tq + min(row0 + kPM, a.Tq));   // last visible position + 1
  const int nb = kend > 0 ? (kend + kPN - 1) / kPN : 0;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0 && nb > 0) {
      tma_prefetch_desc(&tq_hi);
      tma_prefetch_desc(&tk_hi);
      tma_prefetch_desc(&tv_h);
      const int kvrow0 = (b * a.Hkv + hkv) * a.Tmax;
      const float* ksrc = a.ks + (long long)(b * a.Hkv + hkv) * a.Tmax;
      const float* vsrc = a.cv + (long long)(b * a.Hkv + hkv) * a.Tmax;
      mbar_arrive_expect_tx(qfull, 2 * kPM * kPD);
      tma_load_3d(sm + kOffQhi, &tq_hi, qfull, 0, row0, bh);
      tma_load_3d(sm + kOffQlo, &tq_lo, qfull, 0, row0, bh);
      int nk = 0, nsc = 0, nv = 0;
      for (int j = 0; j < nb; ++j) {
        const int s = j % kKSt;
        if (j >= kKSt && !mbar_wait(&kfree[s], (uint32_t)((j / kKSt) - 1) & 1u, abort_flag, a.status, 301)) break;
        uint8_t* kd = sm + kOffK + s * kKStage;
        mbar_arrive_expect_tx(&kfull[s], kKStage);
        tma_load_2d(kd, &tk_hi, &kfull[s], 0, kvrow0 + j * kPN);
        tma_load_2d(kd + kPN * kPD, &tk_lo, &kfull[s], 0, kvrow0 + j * kPN);
        ++nk;
        const int c = j % kScSt;
        if (j >= kScSt && !mbar_wait(&scfree[c], (uint32_t)((j / kScSt) - 1) & 1u, abort_flag, a.status, 302)) break;
        float* sd = reinterpret_cast<float*>(sm + kOffSc + c * kScStage);
        mbar_arrive_expect_tx(&scfull[c], kScStage);
        bulk_load_1d(sd, ksrc + j * kPN, kPN * 4, &scfull[c]);
        bulk_load_1d(sd + kPN, vsrc + j * kPN, kPN * 4, &scfull[c]);
        ++nsc;
        const int v = j % kVSt;
        if (j >= kVSt && !mbar_wait(&vfree[v], (uint32_t)((j / kVSt) - 1) & 1u, abort_flag, a.status, 303)) break;
        uint8_t* vd = sm + kOffV + v * kVStage;
        mbar_arrive_expect_tx(&vfull[v], kVStage);
        tma_load_2d(vd, &tv_h, &vfull[v], 0, kvrow0 + j * kPN);
        tma_load_2d(vd + kPN * 128, &tv_h, &vfull[v], 64, kvrow0 + j * kPN);
        tma_load_2d(vd + 2 * kPN * 128, &tv_l, &vfull[v], 0, kvrow0 + j * kPN);
        tma_load_2d(vd + 3 * kPN * 128, &tv_l, &vfull[v], 64, kvrow0 + j * kPN);
        ++nv;
      }
      // every copy this thread issued lands before the CTA can exit
      drain_wait(qfull, 0u, a.status, 304);
      for (int j = max(0, nk - kKSt); j < nk; ++j) drain_wait(&kfull[j % kKSt], (uint32_t)(j / kKSt) & 1u, a.status, 304);
      for (int j = max(0, nsc - kScSt); j < nsc; ++j)
        drain_wait(&scfull[j % kScSt], (uint32_t)(j / kScSt) & 1u, a.status, 304);
      for (int j = max(0, nv - kVSt); j < nv; ++j) drain_wait(&vfull[j % kVSt], (uint32_t)(j / kVSt) & 1u, a.status, 304);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0 && nb > 0) {
      constexpr uint32_t kIdHH = idesc_i8(kPM, kPN, 1, 1);
      constexpr uint32_t kIdHL = idesc_i8(kPM, kPN, 1, 0);
      constexpr uint32_t kIdLH = idesc_i8(kPM, kPN, 0, 1);
      constexpr uint32_t kIdLL = idesc_i8(kPM, kPN, 0, 0);
      constexpr uint32_t kIdPV = idesc_f16(kPM, kPD, 0, 0, 1);
      const uint32_t qh = smem_u32(sm + kOffQhi), ql = smem_u32(sm + kOffQlo);
      bool ok = mbar_wait(qfull, 0u, abort_flag, a.status, 310);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % kKSt, sb = j & 1;
        if (!mbar_wait(&kfull[s], (uint32_t)(j / kKSt) & 1u, abort_flag, a.status, 311)) return false;
        if (j >= 2 && !mbar_wait(&sfree[sb], (uint32_t)((j >> 1) - 1) & 1u, abort_flag, a.status, 312)) return false;
        tc_fence_after();
        const uint32_t kh = smem_u32(sm + kOffK + s * kKStage), kl = kh + kPN * kPD;
        const uint32_t d = tbase + sb * 192;
#pragma unroll
        for (int ks = 0; ks < kPD / 32; ++ks) {
          const uint32_t o = ks * 32;
          mma_i8(d, kdesc(qh + o), kdesc(kh + o), kIdHH, ks > 0 ? 1u : 0u);
          mma_i8(d + 64, kdesc(qh + o), kdesc(kl + o), kIdHL, ks > 0 ? 1u : 0u);
          mma_i8(d + 64, kdesc(ql + o), kdesc(kh + o), kIdLH, 1u);
          mma_i8(d + 128, kdesc(ql + o), kdesc(kl + o), kIdLL, ks > 0 ? 1u : 0u);
        }
        tc_commit(&sfull[sb]);
        tc_commit(&kfree[s]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int sb = j & 1, v = j % kVSt;
        if (!mbar_wait(&pready[sb], (uint32_t)(j >> 1) & 1u, abort_flag, a.status, 313)) return false;
        if (!mbar_wait(&vfull[v], (uint32_t)(j / kVSt) & 1u, abort_flag, a.status, 314)) return false;
        // the softmax threads have taken the previous block's product out of TMEM
        if (j > 0 && !mbar_wait(ofree, (uint32_t)(j - 1) & 1u, abort_flag, a.status, 316)) return false;
        tc_fence_after();
        const uint32_t ph = smem_u32(sm + kOffP + sb * kPBuf), pr = ph + kPM * kPN * 2;
        const uint32_t vh = smem_u32(sm + kOffV + v * kVStage), vl = vh + 2 * kPN * 128;
        const uint32_t d = tbase + 384;
#pragma unroll
        for (int ks = 0; ks < kPN / 16; ++ks) {
          const uint32_t ao = ks * 32, bo = ks * 2048;
          mma_f16(d, kdesc(ph + ao), vdesc(vh + bo), kIdPV, ks > 0 ? 1u : 0u);
          mma_f16(d, kdesc(ph + ao), vdesc(vl + bo), kIdPV, 1u);
          mma_f16(d, kdesc(pr + ao), vdesc(vh + bo), kIdPV, 1u);
          mma_f16(d, kdesc(pr + ao), vdesc(vl + bo), kIdPV, 1u);
        }
        tc_commit(&vfree[v]);
        tc_commit(&pfree[sb]);
        tc_commit(odone);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; j < nb && ok; ++j) {
        if (j + 1 < nb) ok = issue_qk(j + 1);
        if (ok) ok = issue_pv(j);
      }
      // every MMA issued by this thread completes before TMEM is released
      tc_commit(drain);
      drain_wait(drain, 0u, a.status, 315);
    }
  } else {
    // ------------------------------ softmax warps ------------------------------
    const int sw = warp - kSmWarp0;          // 0 .. kSmWarps-1
    const int qd = warp & 3;                 // TMEM lane quarter this warp may access
    const int hf = sw >> 2;                  // token group of each block, column group of O
    const int r = qd * 32 + lane;            // query row within the tile
    const int tq = row0 + r;
    const bool real = tq < a.Tq;
    const int pos = klen - a.Tq + tq;
    const uint32_t tl_addr = tbase + ((uint32_t)(qd * 32) << 16);
    // logit * log2(e) = fp32(S) * s_k * qcoef; the scores are kept as x' = fp32(S) * s_k and
    // qcoef enters through the row maximum and one FMA per exponent.  qcoef = 0 (an all-zero
    // query row, whose S is 0) or a padding row uses 1 instead: x' is then 0 (or -inf when
    // masked) either way, and no 0 * inf can occur.
    float qcoef = real ? __fmul_rn(__fmul_rn(__ldg(a.qs + (long long)bh * a.Tq + tq), a.scale), kLog2eP) : 1.0f;
    if (!(qcoef > 0.0f)) qcoef = 1.0f;
    const int E = __ldg(a.E + b * a.Hkv + hkv);
    long long* qk_row = (a.qk_out != nullptr && real) ? a.qk_out + ((long long)bh * a.Tq + tq) * a.Tmax : nullptr;
    float* red = reinterpret_cast<float*>(sm + kOffRed);
    float* lsm = reinterpret_cast<float*>(sm + kOffL);
    float m_ref = -INFINITY, l = 0.0f;
    float o_acc[kOCols];                     // this thread's columns of O (FP32, round-to-nearest)
#pragma unroll
    for (int i = 0; i < kOCols; ++i) o_acc[i] = 0.0f;
    float alpha_j = 1.0f;                    // rescale applied at the current block
    const uint32_t ob = tl_addr + 384 + hf * kOCols;
    // O += the product of block jj (complete once PV(jj) has committed), then * alpha
    auto take_block = [&](int jj, float alpha) -> bool {
      if (!mbar_wait(odone, (uint32_t)jj & 1u, abort_flag, a.status, 323)) return false;
      tc_fence_after();
      const bool scaled = __any_sync(0xffffffffu, alpha != 1.0f);
#pragma unroll
      for (int c16 = 0; c16 < kOCols / 16; ++c16) {
        uint32_t o[16];
        tmem_ld16(ob + c16 * 16, o);
        tmem_ld_wait();
        if (scaled) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            o_acc[c16 * 16 + i] = __fmul_rn(__fadd_rn(o_acc[c16 * 16 + i], __uint_as_float(o[i])), alpha);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) o_acc[c16 * 16 + i] = __fadd_rn(o_acc[c16 * 16 + i], __uint_as_float(o[i]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ofree);
      return true;
    };
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      const int sb = j & 1, c = j % kScSt;
      if (!mbar_wait(&sfull[sb], (uint32_t)(j >> 1) & 1u, abort_flag, a.status, 320) ||
          !mbar_wait(&scfull[c], (uint32_t)(j / kScSt) & 1u, abort_flag, a.status, 321)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* scs = reinterpret_cast<const float*>(sm + kOffSc + c * kScStage);   // K scales, then V scales
      float x[kTokPer];
      const uint32_t sbase = tl_addr + sb * 192 + hf * kTokPer;
      // every token of this block visible to every row of the tile: no per-element mask
      const int tlast = j * kPN + kPN - 1;
      const bool full = tlast < klen && (!a.causal || tlast <= klen - a.Tq + row0);
      auto logits = [&](auto mask_c, auto hook_c) {
        constexpr bool kMask = decltype(mask_c)::value, kHook = decltype(hook_c)::value;
#pragma unroll
        for (int q8 = 0; q8 < kTokPer / 8; ++q8) {
          uint32_t rh[8], rx[8], rl[8];
          tmem_ld8(sbase + q8 * 8, rh);
          tmem_ld8(sbase + 64 + q8 * 8, rx);
          tmem_ld8(sbase + 128 + q8 * 8, rl);
          // K scales of these 8 tokens (broadcast shared-memory loads)
          const float4 k0 = *reinterpret_cast<const float4*>(scs + hf * kTokPer + q8 * 8);
          const float4 k1 = *reinterpret_cast<const float4*>(scs + hf * kTokPer + q8 * 8 + 4);
          const float ksv[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int tb = hf * kTokPer + q8 * 8 + i;   // token within the block
            const int t = j * kPN + tb;
            // S = 65536*S_hh + low, low = 256*S_x + S_ll (|low| < 2^31 for head_dim 128);
            // fp32(S) with two roundings: fp32(low), then the FMA (S_hh is exact in fp32)
            const int low = (int)rx[i] * 256 + (int)rl[i];
            const float sf = __fmaf_rn(small_int_to_float((int)rh[i]), 65536.0f, __int2float_rn(low));
            float xv = __fmul_rn(sf, ksv[i]);
            bool vis = true;
            if constexpr (kMask) {
              vis = real && t < klen && (!a.causal || t <= pos);
              if (!vis) xv = -INFINITY;
            }
            if constexpr (kHook) {
              if (vis && qk_row && HEAL_DCHECK(t < a.Tmax && (long long)bh * a.Tq + tq < (long long)a.B * a.Hq * a.Tq,
                                               a.status, 278))
                qk_row[t] = (long long)(int)rh[i] * 65536LL + (long long)low;
            }
            x[q8 * 8 + i] = xv;
          }
        }
      };
      if constexpr (HOOK) {
        logits(std::true_type{}, std::true_type{});
      } else {
        if (full) logits(std::false_type{}, std::false_type{});
        else logits(std::true_type{}, std::false_type{});
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfree[sb]);   // this half of the S buffer is in registers

      // the block's row maximum over both token halves
      float bm;
      {
        float m16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) m16[i] = (kTokPer == 32) ? fmaxf(x[i], x[(i + 16) % kTokPer]) : x[i];
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int i = 0; i < w; ++i) m16[i] = fmaxf(m16[i], m16[i + w]);
        bm = m16[0];
      }
      red[(sb * kGroups + hf) * kPM + r] = bm;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mx[sb * 4 + qd]);
      if (!mbar_wait(&mx[sb * 4 + qd], (uint32_t)(j >> 1) & 1u, abort_flag, a.status, 322)) {
        ok = false;
        break;
      }
      float m_blk = red[(sb * kGroups) * kPM + r];
#pragma unroll
      for (int gi = 1; gi < kGroups; ++gi) m_blk = fmaxf(m_blk, red[(sb * kGroups + gi) * kPM + r]);
      m_blk = __fmul_rn(m_blk, qcoef);          // qcoef > 0: the maximum of fp32(x' * qcoef)
      // lazy maximum: move the reference only when this block exceeds it by more than 2^8
      const bool need = m_blk > m_ref + 8.0f;
      alpha_j = 1.0f;
      if (need) {
        alpha_j = (m_ref == -INFINITY) ? 0.0f : exp2f(m_ref - m_blk);
        m_ref = m_blk;
      }
      l = __fmul_rn(l, alpha_j);

      // P = 2^(x - m_ref) <= 2^8; P' = P * (s_v * 2^E); FP16 P_hi and residual, two tokens a word
      uint32_t phi[kTokPer / 2], prr[kTokPer / 2];
      const float* cvs = scs + kPN;             // s_v * 2^E of the block's tokens (0 past kv_len)
      // a row with no visible token so far keeps m_ref = -inf: subtract 0 instead (P = 0)
      const float msub = (m_ref == -INFINITY) ? 0.0f : m_ref;
      const float nsub = -msub;
      float ls[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int i = 0; i < kTokPer; i += 2) {
        const float p0 = fast_exp2(__fmaf_rn(x[i], qcoef, nsub));
        const float p1 = fast_exp2(__fmaf_rn(x[i + 1], qcoef, nsub));
        ls[(i >> 1) & 3] = __fadd_rn(ls[(i >> 1) & 3], __fadd_rn(p0, p1));
        const float2 c2 = *reinterpret_cast<const float2*>(cvs + hf * kTokPer + i);
        const float q0 = __fmul_rn(p0, c2.x);
        const float q1 = __fmul_rn(p1, c2.y);
        const __half2 hh = __floats2half2_rn(q0, q1);
        const float2 hv = __half22float2(hh);
        const __half2 rr = __floats2half2_rn(__fsub_rn(q0, hv.x), __fsub_rn(q1, hv.y));
        phi[i >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
        prr[i >> 1] = *reinterpret_cast<const uint32_t*>(&rr);
      }
      l = __fadd_rn(l, __fadd_rn(__fadd_rn(ls[0], ls[1]), __fadd_rn(ls[2], ls[3])));
      __syncwarp();
      if (lane == 0) mbar_arrive(&scfree[c]);
      // the P buffer was last read by PV(j-2)
      if (j >= 2 && !mbar_wait(&pfree[sb], (uint32_t)((j >> 1) - 1) & 1u, abort_flag, a.status, 324)) {
        ok = false;
        break;
      }
      // K-major A operand, 128-byte swizzle: row r, 16-byte chunk k at k ^ (r & 7)
      uint8_t* pb = sm + kOffP + sb * kPBuf + r * 128;
#pragma unroll
      for (int cc = 0; cc < kTokPer / 8; ++cc) {
        const int phys = ((hf * (kTokPer / 8) + cc) ^ (r & 7)) * 16;
        *reinterpret_cast<uint4*>(pb + phys) = make_uint4(phi[4 * cc], phi[4 * cc + 1], phi[4 * cc + 2], phi[4 * cc + 3]);
        *reinterpret_cast<uint4*>(pb + kPM * kPN * 2 + phys) =
            make_uint4(prr[4 * cc], prr[4 * cc + 1], prr[4 * cc + 2], prr[4 * cc + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[sb]);
      // the previous block's product, scaled to this block's reference maximum
      if (j > 0 && !take_block(j - 1, alpha_j)) {
        ok = false;
        break;
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    // ---- epilogue: O * 2^-E / l, each warp its 64 columns of 32 rows ----
    if (ok && nb > 0 && !take_block(nb - 1, 1.0f)) ok = false;
    lsm[hf * kPM + r] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(&fin[qd]);
    if (!mbar_wait(&fin[qd], 0u, abort_flag, a.status, 326)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    float L = lsm[r];
#pragma unroll
    for (int gi = 1; gi < kGroups; ++gi) L = __fadd_rn(L, lsm[gi * kPM + r]);
    float* dst = real ? a.out + ((long long)bh * a.Tq + tq) * kPD + hf * kOCols : nullptr;
    if (dst && !HEAL_DCHECK(((long long)bh * a.Tq + tq) * kPD + (hf + 1) * kOCols <= (long long)a.B * a.Hq * a.Tq * kPD,
                            a.status, 279))
      dst = nullptr;
    if (ok && nb > 0) {
      if (dst) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int i = 0; i < kOCols / 4; ++i) {
          float v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            v[u] = L > 0.0f ? __fdiv_rn(mul_pow2_p(o_acc[4 * i + u], -E), L) : 0.0f;
          d4[i] = make_float4(v[0], v[1], v[2], v[3]);
        }
      }
    } else if (ok && dst) {
      // no visible token for this tile (causal with kv_len < Tq): zeros
      float4* d4 = reinterpret_cast<float4*>(dst);
      for (int i = 0; i < kOCols / 4; ++i) d4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

size_t attention_prefill_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tmax) {
  const size_t nk = (size_t)B * Hkv * Tmax * kPD;
  const size_t nq = (size_t)B * Hq * Tq * kPD;
  return 6 * nk + 2 * nq + (size_t)B * Hkv * Tmax * sizeof(float) + (((size_t)B * Hkv * sizeof(int) + 127) & ~(size_t)127);
}

heal_status_t attention_prefill_launch(const int16_t* q, const float* qs, const int16_t* k, const float* ks,
                                       const int16_t* v, const float* vs, int B, int Hq, int Hkv, int Tq,
                                       const int32_t* kv_len, int Tmax, float scale, int causal, float* out,
                                       void* ws, size_t ws_bytes, int64_t* qk_out, cudaStream_t stream) {
  if (ws_bytes < attention_prefill_workspace_bytes(B, Hq, Hkv, Tq, Tmax)) return HEAL_ERR_INVALID_ARGUMENT;
  const long long kv_rows = (long long)B * Hkv * Tmax;
  const long long q_rows = (long long)B * Hq * Tq;
  const int nqt = (Tq + kPM - 1) / kPM;
  if (kv_rows >= (1LL << 31) || q_rows >= (1LL << 31) || (long long)B * Hq * nqt >= (1LL << 31))
    return HEAL_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return HEAL_ERR_CUDA;

  uint8_t* w = static_cast<uint8_t*>(ws);
  const size_t nk = (size_t)kv_rows * kPD, nq = (size_t)q_rows * kPD;
  PlanesArgs pa{};
  pa.q = q;
  pa.k = k;
  pa.v = v;
  pa.vs = vs;
  pa.kv_len = kv_len;
  pa.khi = w;
  pa.klo = w + nk;
  pa.vh = reinterpret_cast<__half*>(w + 2 * nk);
  pa.vl = reinterpret_cast<__half*>(w + 4 * nk);
  pa.qhi = w + 6 * nk;
  pa.qlo = w + 6 * nk + nq;
  pa.cv = reinterpret_cast<float*>(w + 6 * nk + 2 * nq);
  pa.E = reinterpret_cast<int*>(w + 6 * nk + 2 * nq + (size_t)kv_rows * sizeof(float));
  pa.nk8 = (long long)(nk / 8);
  pa.nq8 = (long long)(nq / 8);
  pa.B = B;
  pa.Hkv = Hkv;
  pa.Tmax = Tmax;
  pa.ws = w;
  pa.ws_bytes = (long long)ws_bytes;
  pa.status = device_status_ptr();

  PrefillArgs a{};
  a.qs = qs;
  a.ks = ks;
  a.vs = vs;
  a.kv_len = kv_len;
  a.E = pa.E;
  a.cv = pa.cv;
  a.qk_out = reinterpret_cast<long long*>(qk_out);
  a.out = out;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.Tq = Tq;
  a.Tmax = Tmax;
  a.nqt = nqt;
  a.causal = causal;
  a.scale = scale;
  a.status = device_status_ptr();

  CUtensorMap mq_hi{}, mq_lo{}, mk_hi{}, mk_lo{}, mv_h{}, mv_l{};
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kPD, (cuuint64_t)Tq, (cuuint64_t)B * Hq};
    const cuuint64_t strides[2] = {(cuuint64_t)kPD, (cuuint64_t)Tq * kPD};
    const cuuint32_t box[3] = {kPD, kPM, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    if (!encode_tensor_map(&mq_hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, pa.qhi, dims, strides, box, es,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&mq_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, pa.qlo, dims, strides, box, es,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return HEAL_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kPD, (cuuint64_t)kv_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kPD};
    const cuuint32_t box[2] = {kPD, kPN};
    const cuuint32_t es[2] = {1, 1};
    if (!encode_tensor_map(&mk_hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pa.khi, dims, strides, box, es,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&mk_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pa.klo, dims, strides, box, es,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return HEAL_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kPD, (cuuint64_t)kv_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kPD * 2};
    const cuuint32_t box[2] = {64, kPN};
    const cuuint32_t es[2] = {1, 1};
    if (!encode_tensor_map(&mv_h, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pa.vh, dims, strides, box, es,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&mv_l, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pa.vl, dims, strides, box, es,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return HEAL_ERR_CUDA;
  }

  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HEAL_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(heal_attn_prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(heal_attn_prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem) !=
            cudaSuccess)
      return HEAL_ERR_CUDA;
    attr_set[dev] = true;
  }
  const long long chunks = pa.nk8 > pa.nq8 ? pa.nk8 : pa.nq8;
  long long gx = (chunks + 255) / 256;
  if (gx > (long long)sms * 4) gx = (long long)sms * 4;
  if (gx < (long long)B * Hkv) gx = (long long)B * Hkv;
  cudaError_t e = launch_pdl(heal_attn_planes_kernel, dim3((unsigned)gx, 4), dim3(256), 0, stream, pa);
  if (e != cudaSuccess) return HEAL_ERR_CUDA;
  if (qk_out)
    e = launch_pdl(heal_attn_prefill_kernel<true>, dim3((unsigned)(B * Hq * nqt)), dim3(kPThreads), (size_t)kPSmem,
                   stream, mq_hi, mq_lo, mk_hi, mk_lo, mv_h, mv_l, a);
  else
    e = launch_pdl(heal_attn_prefill_kernel<false>, dim3((unsigned)(B * Hq * nqt)), dim3(kPThreads), (size_t)kPSmem,
                   stream, mq_hi, mq_lo, mk_hi, mk_lo, mv_h, mv_l, a);
  if (e != cudaSuccess) return HEAL_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

}  // namespace heal
