// gemm_tc.cu -- error-compensated GEMM on sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
// Method (authors' v2 abstract; gist.science technical summary, section 2.B): each FP32
// operand x is split into a 16-bit primary value and a 16-bit residual,
//     hi = r16(x),  lo = r16((x - hi) * 2^L)          (L = 11 for FP16, 0 for BF16)
// and C = A.B is synthesised from three 16-bit products with FP32 accumulation,
//     C ~= Ah.Bh + 2^-L (Ah.Bl + Al.Bh).
//
// Kernel structure (one persistent CTA per SM, 12 warps; 13 for the tiles with BN <= 32):
//   warp 0      TMA producer: FP32 tiles of both operands, 128-byte swizzled, into a
//               ring of shared-memory stages (one stage = 64 values of K).
//   warp 1      MMA issuer (one thread): per stage, the two correction products into a
//               fresh TMEM accumulator, then Ah.Bh with scale-input-d = L, which scales
//               the corrections by 2^-L as it adds the main product, then the rest of
//               Ah.Bh.  Two TMEM accumulator buffers for the 128-wide tile, four for the
//               skinny tiles; with BN <= 32 a second issuer (warp 12) takes every other
//               work unit.
//   warps 2-7   split warps: read the FP32 stage, write hi and lo back into the same
//               shared memory in the UMMA 128-byte-swizzle canonical layout, fence the
//               async proxy and release the stage to the MMA issuer.  (No split pass
//               goes through HBM.)
//   warps 8-11  epilogue: drain each 64-wide K chunk from TMEM and add it to the running
//               FP32 sum in registers (round-to-nearest, ascending chunk order), then
//               store C.  In split-K mode every chunk value goes to a workspace instead
//               (at BN = 64 through shared memory and a TMA store), and a reduce kernel
//               adds them in the same order.  In chain mode (a
//               cluster of S CTAs per tile, each owning a contiguous run of chunks) every
//               chunk keeps its own TMEM accumulator; at the end the running FP32 sum is
//               handed from CTA to CTA through distributed shared memory in ascending chunk
//               order, and the last CTA of the cluster stores C.
// Because every chunk value comes from the same sequence of tensor-core instructions and
// chunk values are added in a fixed order, C is identical bit for bit across runs, tile
// shapes, operand swapping and split-K.
//
// Operand roles inside the kernel: "kernel-A" supplies the 128 MMA rows (TMEM lanes),
// "kernel-B" the BN MMA columns.  Normal mode: kernel-A = A, kernel-B = B^T.  Swapped mode
// (skinny M): kernel-A = B^T (weights), kernel-B = A, and C is written transposed.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "heal_internal.h"
#include "heal_ptx.cuh"
#include "heal_split.cuh"

namespace heal {

constexpr int kBM = 128;   // MMA M: rows of kernel-A per tile (= TMEM lanes)
constexpr int kBK = 64;    // K per stage = one accumulation chunk
constexpr int kSplitWarp0 = 2, kNumEpiWarps = 4;

// Warp roles per tile width: warp 0 TMA, warp 1 MMA, then the split warps, then four
// epilogue warps (which must start at a multiple of 4 so that warp % 4 names the TMEM lane
// quarter).  Six split warps for every tile width (ten measured no faster on the skinny
// decode tiles, whose time goes elsewhere).
// The skinny tiles with BN <= 32 have a second MMA issuer, one warp after the epilogue
// warps: an N <= 32 MMA is short, so one thread's issue rate (tens of cycles per
// tcgen05.mma plus the per-stage waits and commits) bounds these tiles; the two issuers take
// alternate work units, each with its own TMEM accumulator buffer (chain mode keeps one
// issuer).  BN = 64 keeps twelve warps: with a thirteenth, four warps share one SM
// sub-partition and its 64-column epilogue would be held to 128 registers.
template <int BN>
struct Roles {
  static constexpr int kSplitWarps = 6;
  static constexpr int kEpiWarp0 = kSplitWarp0 + kSplitWarps;
  static constexpr int kMmaIssuers = BN <= 32 ? 2 : 1;
  static constexpr int kMma2Warp = kEpiWarp0 + kNumEpiWarps;   // the second issuer's warp
  static constexpr int kThreads = (kEpiWarp0 + kNumEpiWarps + kMmaIssuers - 1) * 32;
  static_assert(kEpiWarp0 % 4 == 0, "epilogue warps must start at a lane-quarter boundary");
};

struct GemmArgs {
  int Mk, Nk, K;            // kernel-space rows of kernel-A, rows of kernel-B, reduction
  int tiles_m, tiles_n, num_chunks;
  int splitk;               // 1: write chunk partials to ws
  int chain;                // S >= 2: chain mode, S CTAs (one cluster) per tile, 0 otherwise
  int tmem_cols;            // TMEM columns this kernel allocates (power of two, 32 .. 512)
  float* out;
  long long out_si, out_sj; // element (i, j) -> out[i*si + j*sj]
  float* ws;                // [num_chunks][Nk][Mk] chunk values (split-K mode)
  const int8_t* chan_exp;   // nullable, [K]
  int expA_sign, expB_sign; // +1 / -1: which operand gets 2^+e and which 2^-e
  int static_op;            // 0: none; 1: kernel-A, 2: kernel-B is not written by the kernels
                            // before this one (its first stages may be requested early)
  unsigned int* status;     // device status word
  long long out_extent;      // elements of `out` the call may write (debug-build checks)
  int ws_tma;               // split K, BN = 64: chunk tiles go to ws by TMA store (map in the B-lo slot)
  long long ws_elems;       // FP32 elements of the workspace (debug-build checks)
};

template <int BN>
struct Cfg {
  static constexpr int kABytes = kBM * kBK * 4;             // 32 KB of FP32
  static constexpr int kBBytes = BN * kBK * 4;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (216 * 1024) / kStageBytes > 8 ? 8 : (216 * 1024) / kStageBytes;
  // TMEM accumulator buffers: four for the skinny tiles (the MMA issuers run up to three
  // work units ahead of the epilogue), two for the 128-wide tile
  static constexpr int kAccBufs = BN <= 64 ? 4 : 2;
  static constexpr int kTmemCols = (kAccBufs * BN) <= 32 ? 32 : (kAccBufs * BN) <= 64 ? 64 : (kAccBufs * BN) <= 128 ? 128
                                 : (kAccBufs * BN) <= 256 ? 256 : 512;
  // chain mode (BN <= 32): the running sum a predecessor CTA hands over, 128 rows x BN FP32
  static constexpr int kSumBytes = BN <= 32 ? kBM * BN * 4 : 0;
  // split K at BN = 64: one chunk tile (BN rows x 128 FP32) staged for a TMA store to the
  // workspace (the 64-column stores per thread otherwise bound the epilogue)
  static constexpr int kStoreBytes = BN == 64 ? kBM * BN * 4 : 0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kSumBytes + kStoreBytes + 1024 /*barriers*/ + 1024 /*align*/;
  static_assert(kStages >= 2, "at least two stages");
};

// ---------------------------------------------------------------------------------
// Work iteration shared by every role: (tile, chunk) pairs in a fixed order.
//   full-K mode : tiles blockIdx.x, +gridDim.x, ...; chunks 0..num_chunks-1 per tile
//   split-K mode: a contiguous slice of the flattened (tile, chunk) sequence
// ---------------------------------------------------------------------------------
struct WorkIter {
  int tile, chunk, u, u_end, ntiles, nc, splitk;
  int step, dtile, dchunk;   // split K: chunk-major units dealt round-robin
  __device__ WorkIter(const GemmArgs& a) {
    ntiles = a.tiles_m * a.tiles_n;
    nc = a.num_chunks;
    splitk = a.splitk || a.chain;
    if (a.chain) {
      // one tile per cluster of S CTAs; CTA rank r owns chunks [r*nc/S, (r+1)*nc/S)
      const int S = a.chain, t = blockIdx.x / S, r = blockIdx.x % S;
      u = t * nc + (r * nc) / S;
      u_end = t * nc + ((r + 1) * nc) / S;
      tile = t;
      chunk = u - t * nc;
      step = 0;
      dtile = dchunk = 0;
    } else if (splitk) {
      // unit u = (chunk u / ntiles, tile u % ntiles); CTA c takes u = c, c + grid, ...: the
      // CTAs working at the same time cover every tile of the same few chunks, i.e. whole
      // rows of the weights, a contiguous region of memory
      u = blockIdx.x;
      u_end = ntiles * nc;
      step = gridDim.x;
      dtile = step % ntiles;
      dchunk = step / ntiles;
      tile = u % ntiles;
      chunk = u / ntiles;
    } else {
      tile = blockIdx.x;
      chunk = 0;
      u = 0;
      u_end = 0;
      step = dtile = dchunk = 0;
    }
  }
  __device__ bool valid() const { return splitk ? (u < u_end) : (tile < ntiles); }
  __device__ void advance() {
    if (splitk && step == 0) {   // chain mode: consecutive chunks of one tile
      ++u;
      if (++chunk == nc) {
        chunk = 0;
        ++tile;
      }
    } else if (splitk) {         // tile = u % ntiles, chunk = u / ntiles, kept incrementally
      u += step;
      tile += dtile;
      chunk += dchunk;
      if (tile >= ntiles) {
        tile -= ntiles;
        ++chunk;
      }
    } else if (++chunk == nc) {
      chunk = 0;
      tile += gridDim.x;
    }
  }
};

// Tile raster: groups of 8 kernel-A row tiles, column tiles inside a group.
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int& tm, int& tn) {
  if (tiles_n == 1) {   // one column of tiles (the skinny kernels): the raster is the identity
    tm = tile;
    tn = 0;
    return;
  }
  constexpr int GM = 8;
  const int group = GM * tiles_n;
  const int g = tile / group;
  const int first_m = g * GM;
  const int gm = min(tiles_m - first_m, GM);
  const int local = tile - g * group;
  tm = first_m + local % gm;
  tn = local / gm;
}

// ---------------------------------------------------------------------------------
// TMA of one operand tile (R rows x 64 K) into a stage.
//   K-major  (K contiguous) : two boxes {32 K, R rows} -> [0, R*128) and [R*128, R*256)
//   MN-major (rows contiguous): R/32 boxes {32 rows, 64 K} -> b*8192
//   16-bit pre-split input   : hi/lo boxes of 64 values that land exactly where the
//                              in-place split would have written them (PRE = 1), or
//                              the hi boxes alone for a 16-bit operand (PRE = 2).
// ---------------------------------------------------------------------------------
template <int R, bool MN, int PRE>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, const CUtensorMap* map_lo,
                                             uint64_t* bar, int row0, int k0) {
  if constexpr (PRE == 0) {
    if constexpr (!MN) {
      tma_load_2d(dst, map, bar, k0, row0);
      tma_load_2d(dst + R * 128, map, bar, k0 + 32, row0);
    } else {
#pragma unroll
      for (int b = 0; b < R / 32; ++b) tma_load_2d(dst + b * 8192, map, bar, row0 + 32 * b, k0);
    }
  } else {
    if constexpr (!MN) {
      tma_load_2d(dst, map, bar, k0, row0);                                   // hi: R rows x 64 values
      if constexpr (PRE == 1) tma_load_2d(dst + R * 128, map_lo, bar, k0, row0);  // lo
    } else {
#pragma unroll
      for (int p = 0; p < R / 64; ++p) {
        tma_load_2d(dst + (2 * p) * 8192, map, bar, row0 + 64 * p, k0);
        if constexpr (PRE == 1) tma_load_2d(dst + (2 * p + 1) * 8192, map_lo, bar, row0 + 64 * p, k0);
      }
    }
  }
}

// The same loads with an L2 cache-policy hint: evict-first for an operand streamed once
// (the weights of the split-K decode kernels, so that they do not push the chunk workspace
// out of L2), evict-last for one every column stripe reuses (A in the CTA-pair kernel).
template <int R, bool MN, int PRE>
__device__ __forceinline__ void load_operand_once(uint8_t* dst, const CUtensorMap* map, const CUtensorMap* map_lo,
                                                  uint64_t* bar, int row0, int k0, uint64_t pol) {
  if constexpr (PRE == 0) {
    if constexpr (!MN) {
      tma_load_2d_hint(dst, map, bar, k0, row0, pol);
      tma_load_2d_hint(dst + R * 128, map, bar, k0 + 32, row0, pol);
    } else {
#pragma unroll
      for (int b = 0; b < R / 32; ++b) tma_load_2d_hint(dst + b * 8192, map, bar, row0 + 32 * b, k0, pol);
    }
  } else {
    if constexpr (!MN) {
      tma_load_2d_hint(dst, map, bar, k0, row0, pol);
      if constexpr (PRE == 1) tma_load_2d_hint(dst + R * 128, map_lo, bar, k0, row0, pol);
    } else {
#pragma unroll
      for (int p = 0; p < R / 64; ++p) {
        tma_load_2d_hint(dst + (2 * p) * 8192, map, bar, row0 + 64 * p, k0, pol);
        if constexpr (PRE == 1) tma_load_2d_hint(dst + (2 * p + 1) * 8192, map_lo, bar, row0 + 64 * p, k0, pol);
      }
    }
  }
}

// ---------------------------------------------------------------------------------
// In-place split of one 2 KB region pair by one warp.
// src0/src1 each hold one 128-byte-swizzled atom of 8 rows x 32 FP32 values; together
// they are 8 rows x 64 values.  Afterwards src0 holds the 16-bit hi atom (8 rows x 64)
// and src1 the lo atom, both in the 128-byte-swizzle canonical layout.
// Lane -> (atom row = lane & 7, quarter = lane >> 3): conflict-free 16-byte accesses.
// kb: K index of the region's first value (K-major) or first row (MN-major), used for
// the optional channel exponents; values at K >= K are TMA zero fill and stay zero.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Load half: this lane's 16 FP32 values (two 16-byte pieces of each atom).
__device__ __forceinline__ void split_load(const uint8_t* src0, const uint8_t* src1, int lane, float (&v)[16]) {
  const int row = lane & 7, q = lane >> 3;
  const uint8_t* r0 = src0 + row * 128;
  const uint8_t* r1 = src1 + row * 128;
  *reinterpret_cast<float4*>(&v[0]) = *reinterpret_cast<const float4*>(r0 + (((2 * q) ^ row) << 4));
  *reinterpret_cast<float4*>(&v[4]) = *reinterpret_cast<const float4*>(r0 + (((2 * q + 1) ^ row) << 4));
  *reinterpret_cast<float4*>(&v[8]) = *reinterpret_cast<const float4*>(r1 + (((2 * q) ^ row) << 4));
  *reinterpret_cast<float4*>(&v[12]) = *reinterpret_cast<const float4*>(r1 + (((2 * q + 1) ^ row) << 4));
}

// Store half: optional channel exponents, the split, and the hi / lo 16-byte pieces.  The
// caller has synchronised the warp after every lane's split_load of this region.
template <int FMT, bool MN>
__device__ __forceinline__ void split_store(uint8_t* src0, uint8_t* src1, int lane, float (&v)[16],
                                            const int8_t* chan_exp, int exp_sign, int kb, int K) {
  const int row = lane & 7, q = lane >> 3;
  uint8_t* r0 = src0 + row * 128;
  uint8_t* r1 = src1 + row * 128;
  if (chan_exp != nullptr) {
    if constexpr (MN) {
      // every value of this lane has K index kb + row
      const int k = kb + row;
      const float s = k < K ? pow2f(exp_sign * (int)__ldg(chan_exp + k)) : 0.0f;   // beyond K: TMA zero fill
#pragma unroll
      for (int t = 0; t < 16; ++t) v[t] = __fmul_rn(v[t], s);
    } else {
      // K index of value t: kb + 8q + t (t < 8), kb + 32 + 8q + (t - 8)
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const int k = kb + (t < 8 ? 8 * q + t : 32 + 8 * q + (t - 8));
        if (k < K) v[t] = __fmul_rn(v[t], pow2f(exp_sign * (int)__ldg(chan_exp + k)));
      }
    }
  }
  uint4 h0, h1, l0, l1;
  h0.x = split2<FMT>(v[0], v[1], l0.x);
  h0.y = split2<FMT>(v[2], v[3], l0.y);
  h0.z = split2<FMT>(v[4], v[5], l0.z);
  h0.w = split2<FMT>(v[6], v[7], l0.w);
  h1.x = split2<FMT>(v[8], v[9], l1.x);
  h1.y = split2<FMT>(v[10], v[11], l1.y);
  h1.z = split2<FMT>(v[12], v[13], l1.z);
  h1.w = split2<FMT>(v[14], v[15], l1.w);
  *reinterpret_cast<uint4*>(r0 + ((q ^ row) << 4)) = h0;
  *reinterpret_cast<uint4*>(r0 + (((4 + q) ^ row) << 4)) = h1;
  *reinterpret_cast<uint4*>(r1 + ((q ^ row) << 4)) = l0;
  *reinterpret_cast<uint4*>(r1 + (((4 + q) ^ row) << 4)) = l1;
}

// One warp splits one 2 KB region pair in place.
template <int FMT, bool MN>
__device__ __forceinline__ void split_pair(uint8_t* src0, uint8_t* src1, int lane, const int8_t* chan_exp,
                                           int exp_sign, int kb, int K) {
  float v[16];
  split_load(src0, src1, lane, v);
  __syncwarp();   // every lane has read the region before any lane overwrites it
  split_store<FMT, MN>(src0, src1, lane, v, chan_exp, exp_sign, kb, K);
}

// Region pair t of an operand tile with R rows (t in [0, R/8)).
template <int R, bool MN>
__device__ __forceinline__ void pair_addr(uint8_t* base, int t, uint8_t*& s0, uint8_t*& s1, int& kb_off) {
  if constexpr (!MN) {
    s0 = base + t * 1024;
    s1 = base + R * 128 + t * 1024;
    kb_off = 0;
  } else {
    const int p = t >> 3, j = t & 7;
    s0 = base + (2 * p) * 8192 + j * 1024;
    s1 = base + (2 * p + 1) * 8192 + j * 1024;
    kb_off = 8 * j;
  }
}

// Shared-memory descriptors of the hi / lo tiles of an operand with R rows.
template <int R, bool MN>
struct OperandDesc {
  static __device__ __forceinline__ uint64_t hi(uint32_t base) {
    return MN ? smem_desc_sw128(base, 16384, 1024) : smem_desc_sw128(base, 16, 1024);
  }
  static __device__ __forceinline__ uint64_t lo(uint32_t base) {
    return MN ? smem_desc_sw128(base + 8192, 16384, 1024) : smem_desc_sw128(base + R * 128, 16, 1024);
  }
  // advance by one K=16 step (descriptor address field counts 16-byte units)
  static constexpr uint64_t kStep = MN ? (2048 >> 4) : (32 >> 4);
};

// ---------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------
// A_PRE / B_PRE: 0 FP32 split in the kernel, 1 pre-split hi + lo, 2 a 16-bit operand with
// no residual (its correction product is absent: the two-product form).
template <int BN, bool A_MN, bool B_MN, int FMT, bool CORR_SWAP, int A_PRE, int B_PRE>
__global__ void __launch_bounds__(Roles<BN>::kThreads, 1)
    heal_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA_lo,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB_lo,
                     const GemmArgs args) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  constexpr int kNumSplitWarps = Roles<BN>::kSplitWarps;
  constexpr int kEpiWarp0 = Roles<BN>::kEpiWarp0;
  // bytes that land in a stage (a 16-bit-only operand fills only its hi half)
  constexpr uint32_t kStageTx = C::kStageBytes - (A_PRE == 2 ? C::kABytes / 2 : 0) - (B_PRE == 2 ? C::kBBytes / 2 : 0);
  constexpr bool kHasALo = A_PRE != 2, kHasBLo = B_PRE != 2;
  constexpr int kLoShift = FMT == 0 ? 11 : 0;
  constexpr uint32_t kIdesc = idesc_f16(kBM, BN, FMT, A_MN ? 1 : 0, B_MN ? 1 : 0);

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment of the shared-window address (128-byte swizzle atoms)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  float* sum_buf = reinterpret_cast<float*>(smem + S * C::kStageBytes);   // chain mode: [128 rows][BN]
  float* out_stage = reinterpret_cast<float*>(smem + S * C::kStageBytes + C::kSumBytes);   // [BN][128] (BN = 64)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kSumBytes + C::kStoreBytes);
  uint64_t* full = bars;                 // TMA -> split       (tx bytes)
  uint64_t* split_done = bars + S;       // split -> MMA       (all split threads arrive)
  uint64_t* empty = bars + 2 * S;        // MMA -> TMA         (tcgen05.commit)
  constexpr int NB = C::kAccBufs;
  uint64_t* acc_full = bars + 3 * S;          // MMA -> epilogue    (tcgen05.commit)
  uint64_t* acc_empty = bars + 3 * S + NB;    // epilogue -> MMA    (128 arrivals)
  uint64_t* mma_done = bars + 3 * S + 2 * NB; // MMA drain on exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 2 * NB + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 3 * S + 2 * NB + 2);
  uint64_t* chain_bar = bars + 3 * S + 2 * NB + 3; // chain mode: the predecessor's running sum has landed

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();   // a following reduce kernel may be scheduled; it waits for us

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&split_done[s], kNumSplitWarps * 32);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kNumEpiWarps * 32);
    }
    mbar_init(mma_done, args.chain ? 1 : Roles<BN>::kMmaIssuers);
    mbar_init(chain_bar, kNumEpiWarps * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, (uint32_t)args.tmem_cols);
    tmem_relinquish();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (A_PRE == 1) tma_prefetch_desc(&tmA_lo);
    if (B_PRE == 1) tma_prefetch_desc(&tmB_lo);
  }
  tc_fence_before();
  __syncthreads();
  if (args.chain) cluster_sync_all();   // every CTA's chain barrier is initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  constexpr bool kRegSplit = (BN == 128);   // epilogue holds 128 FP32 sums per thread
  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if constexpr (kRegSplit) setmaxnreg_dec<96>();
    if (lane == 0) {
      // Programmatic dependent launch: this grid may start while the kernel before it is
      // still running.  An operand the caller declared static is requested for the first
      // stages right away; everything else waits for the preceding grid to finish.
      int pre = 0;
      const uint64_t pol = l2_policy_evict_first();
      // split-K and chain modes: kernel-A (the weights) is read exactly once
      auto load_a = [&](uint8_t* st, uint64_t* bar, int tm, int k0) {
        if (args.splitk || args.chain) load_operand_once<kBM, A_MN, A_PRE>(st, &tmA, &tmA_lo, bar, tm * kBM, k0, pol);
        else load_operand<kBM, A_MN, A_PRE>(st, &tmA, &tmA_lo, bar, tm * kBM, k0);
      };
      if (args.static_op != 0) {
        for (WorkIter w(args); w.valid() && pre < S; w.advance(), ++pre) {
          int tm, tn;
          tile_coords(w.tile, args.tiles_m, args.tiles_n, tm, tn);
          const int k0 = w.chunk * kBK;
          uint8_t* st = stages + pre * C::kStageBytes;
          mbar_arrive_expect_tx(&full[pre], kStageTx);
          if (args.static_op == 1) load_a(st, &full[pre], tm, k0);
          else load_operand<BN, B_MN, B_PRE>(st + C::kABytes, &tmB, &tmB_lo, &full[pre], tn * BN, k0);
        }
      }
      pdl_wait_prerequisites();
      int it = 0;
      for (WorkIter w(args); w.valid(); w.advance(), ++it) {
        const int s = it % S;
        const uint32_t ph = (uint32_t)(it / S) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, args.status, 100)) break;
        int tm, tn;
        tile_coords(w.tile, args.tiles_m, args.tiles_n, tm, tn);
        const int k0 = w.chunk * kBK;
        uint8_t* st = stages + s * C::kStageBytes;
        if (it >= pre) mbar_arrive_expect_tx(&full[s], kStageTx);
        if (it >= pre || args.static_op != 1) load_a(st, &full[s], tm, k0);
        if (it >= pre || args.static_op != 2)
          load_operand<BN, B_MN, B_PRE>(st + C::kABytes, &tmB, &tmB_lo, &full[s], tn * BN, k0);
      }
      // Do not leave the CTA with copies in flight: wait (bounded) for the last fill of
      // every stage that was issued.
      for (int j = 0; j < S && j < it; ++j) {
        const int jt = it - 1 - j;
        volatile int dummy = 0;
        mbar_wait(&full[jt % S], (uint32_t)(jt / S) & 1u, &dummy, args.status, 101);
      }
    }
  } else if (warp == 1 || (Roles<BN>::kMmaIssuers == 2 && warp == Roles<BN>::kMma2Warp)) {
    // ------------------------------ MMA issuer(s) ------------------------------
    // With two issuers, issuer q takes the work units it with it % 2 == q (TMEM buffers
    // it % NB of that parity); every unit's MMAs come from one thread and its commits track
    // exactly them.
    if constexpr (kRegSplit) setmaxnreg_dec<96>();
    const int nis = args.chain ? 1 : Roles<BN>::kMmaIssuers;
    const int q = warp == 1 ? 0 : 1;
    if (lane == 0 && q < nis) {
      int it = 0;
      for (WorkIter w(args); w.valid(); w.advance(), ++it) {
        if (nis == 2 && (it & 1) != q) continue;
        const int s = it % S;
        const uint32_t ph = (uint32_t)(it / S) & 1u;
        const int b = it % NB;
        const uint32_t aph = (uint32_t)(it / NB) & 1u;
        if (!mbar_wait(&split_done[s], ph, abort_flag, args.status, 110)) break;
        if (!args.chain && !mbar_wait(&acc_empty[b], aph ^ 1u, abort_flag, args.status, 111)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(stages + s * C::kStageBytes);
        const uint32_t sb = sa + C::kABytes;
        const uint64_t a_hi = OperandDesc<kBM, A_MN>::hi(sa), a_lo = OperandDesc<kBM, A_MN>::lo(sa);
        const uint64_t b_hi = OperandDesc<BN, B_MN>::hi(sb), b_lo = OperandDesc<BN, B_MN>::lo(sb);
        constexpr uint64_t dA = OperandDesc<kBM, A_MN>::kStep, dB = OperandDesc<BN, B_MN>::kStep;
        // chain mode: every chunk of this CTA has its own accumulator columns
        const uint32_t d = tmem_base + (uint32_t)((args.chain ? it : b) * BN);
        // corrections first: Ah.Bl then Al.Bh in the caller's operand order (a 16-bit
        // operand has no residual, so its correction product is absent)
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j) {
          uint32_t acc_in = j > 0 ? 1u : 0u;
          if constexpr (!CORR_SWAP) {
            if constexpr (kHasBLo) { mma_f16(d, a_hi + j * dA, b_lo + j * dB, kIdesc, acc_in); acc_in = 1u; }
            if constexpr (kHasALo) mma_f16(d, a_lo + j * dA, b_hi + j * dB, kIdesc, acc_in);
          } else {
            if constexpr (kHasALo) { mma_f16(d, a_lo + j * dA, b_hi + j * dB, kIdesc, acc_in); acc_in = 1u; }
            if constexpr (kHasBLo) mma_f16(d, a_hi + j * dA, b_lo + j * dB, kIdesc, acc_in);
          }
        }
        // main product; its first step scales the corrections by 2^-L
        mma_f16_scale_d<kLoShift>(d, a_hi, b_hi, kIdesc);
#pragma unroll
        for (int j = 1; j < kBK / 16; ++j) mma_f16(d, a_hi + j * dA, b_hi + j * dB, kIdesc, 1u);
        tc_commit(&empty[s]);
        if (!args.chain) tc_commit(&acc_full[b]);
      }
      if (args.chain) tc_commit(&acc_full[0]);   // every chunk of this CTA is in TMEM
      // drain: every MMA issued by this thread has completed before TMEM is released
      tc_commit(mma_done);
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, &dummy, args.status, 112);
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------ split warps ------------------------------
    if constexpr (kRegSplit) setmaxnreg_dec<96>();
    pdl_wait_prerequisites();   // chan_exp may come from the preceding kernel
    const int sw = warp - kSplitWarp0;
    constexpr int kPairsA = kBM / 8, kPairsB = BN / 8;
    int it = 0;
    for (WorkIter w(args); w.valid(); w.advance(), ++it) {
      const int s = it % S;
      const uint32_t ph = (uint32_t)(it / S) & 1u;
      if (!mbar_wait(&full[s], ph, abort_flag, args.status, 120)) break;
      uint8_t* st = stages + s * C::kStageBytes;
      const int k0 = w.chunk * kBK;
      constexpr int kFirst = A_PRE ? kPairsA : 0;
      constexpr int kLast = B_PRE ? kPairsA : kPairsA + kPairsB;
      for (int t = kFirst + sw; t < kLast; t += kNumSplitWarps) {
        uint8_t *s0, *s1;
        int kboff;
        if (t < kPairsA) {
          pair_addr<kBM, A_MN>(st, t, s0, s1, kboff);
          split_pair<FMT, A_MN>(s0, s1, lane, args.chan_exp, args.expA_sign, k0 + kboff, args.K);
        } else {
          pair_addr<BN, B_MN>(st + C::kABytes, t - kPairsA, s0, s1, kboff);
          split_pair<FMT, B_MN>(s0, s1, lane, args.chan_exp, args.expB_sign, k0 + kboff, args.K);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&split_done[s]);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    if constexpr (kRegSplit) setmaxnreg_inc<240>();
    pdl_wait_prerequisites();   // C and the workspace may still be read by the preceding kernel
    const int quarter = warp & 3;            // TMEM lanes this warp may access
    const int i_local = quarter * 32 + lane; // tile row
    float acc[BN];
#pragma unroll
    for (int t = 0; t < BN; ++t) acc[t] = 0.0f;
    if constexpr (BN <= 32) {
      if (args.chain) {
        // ---- chain mode: add this CTA's chunk values onto the predecessor's running sum,
        // in ascending chunk order, and hand the sum on (or store C at the end of K) ----
        const WorkIter w0(args);
        const int nloc = w0.u_end - w0.u;
        const int r = (int)(blockIdx.x % (unsigned)args.chain);
        bool ok = nloc > 0 && mbar_wait(&acc_full[0], 0u, abort_flag, args.status, 140);
        if (ok) {
          tc_fence_after();
          if (r > 0) {
            ok = mbar_wait_cluster(chain_bar, 0u, abort_flag, args.status, 141);
            if (ok) {
#pragma unroll
              for (int t = 0; t < BN; t += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(sum_buf + i_local * BN + t);
                acc[t] = v4.x;
                acc[t + 1] = v4.y;
                acc[t + 2] = v4.z;
                acc[t + 3] = v4.w;
              }
            }
          }
        }
        if (ok) {
          const uint32_t tq = tmem_base + ((uint32_t)(quarter * 32) << 16);
          for (int k = 0; k < nloc; ++k) {
            const bool first = (r == 0 && k == 0);
#pragma unroll
            for (int c = 0; c < BN / 16; ++c) {
              uint32_t v[16];
              tmem_ld16(tq + (uint32_t)(k * BN + c * 16), v);
              tmem_ld_wait();
#pragma unroll
              for (int t = 0; t < 16; ++t) {
                const float dv = __uint_as_float(v[t]);
                acc[c * 16 + t] = first ? dv : __fadd_rn(acc[c * 16 + t], dv);
              }
            }
          }
          tc_fence_before();
          int tm, tn;
          tile_coords(w0.tile, args.tiles_m, args.tiles_n, tm, tn);
          const int gi = tm * kBM + i_local;
          if (r + 1 < args.chain) {
            // into the successor's sum buffer (same offset in its shared memory), then
            // release-arrive on its chain barrier
            const uint32_t dst = mapa_shared(smem_u32(sum_buf + i_local * BN), (uint32_t)(r + 1));
#pragma unroll
            for (int t = 0; t < BN; t += 4) st_shared_cluster_v4(dst + (uint32_t)(t * 4), acc[t], acc[t + 1], acc[t + 2], acc[t + 3]);
            mbar_arrive_cluster(mapa_shared(smem_u32(chain_bar), (uint32_t)(r + 1)));
          } else if (gi < args.Mk) {
#pragma unroll
            for (int t = 0; t < BN; ++t) {
              const int gj = tn * BN + t;
              const long long o = (long long)gi * args.out_si + (long long)gj * args.out_sj;
              if (gj < args.Nk && HEAL_DCHECK(o < args.out_extent, args.status, 150)) args.out[o] = acc[t];
            }
          }
        }
        (void)ok;
      }
    }
    int it = 0;
    bool ok = true;
    for (WorkIter w(args); !args.chain && w.valid(); w.advance(), ++it) {
      const int b = it % NB;
      const uint32_t aph = (uint32_t)(it / NB) & 1u;
      if (!mbar_wait(&acc_full[b], aph, abort_flag, args.status, 130)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int tm, tn;
      tile_coords(w.tile, args.tiles_m, args.tiles_n, tm, tn);
      const int gi = tm * kBM + i_local;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN);
      if (!args.splitk) {
        const bool first = (w.chunk == 0);
#pragma unroll
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(taddr + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float dv = __uint_as_float(r[t]);
            acc[c * 16 + t] = first ? dv : __fadd_rn(acc[c * 16 + t], dv);
          }
        }
      } else {
        // all of the chunk's columns are loaded before one wait, and the TMEM buffer is
        // handed back before the stores
        float* wsc = args.ws + (size_t)w.chunk * args.Nk * args.Mk;
        uint32_t r[BN / 16][16];
#pragma unroll
        for (int c = 0; c < BN / 16; ++c) tmem_ld16(taddr + c * 16, r[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
        if constexpr (C::kStoreBytes > 0 && B_PRE == 0) {
          if (args.ws_tma) {
            // the chunk tile through shared memory and one TMA store (the workspace's map
            // rides in the kernel-B lo slot: kernel-B, the activations, is never pre-split
            // here).  The previous tile's store must have read the staging buffer first.
            const bool issuer = (warp == kEpiWarp0 && lane == 0);
            if (issuer) bulk_wait_group_read0();
            named_bar_sync(1, kNumEpiWarps * 32);
#pragma unroll
            for (int c = 0; c < BN / 16; ++c)
#pragma unroll
              for (int t = 0; t < 16; ++t) out_stage[(c * 16 + t) * kBM + i_local] = __uint_as_float(r[c][t]);
            fence_proxy_async_smem();
            named_bar_sync(1, kNumEpiWarps * 32);
            if (issuer && HEAL_DCHECK(w.chunk < args.num_chunks, args.status, 156)) {
              tma_store_3d(&tmB_lo, out_stage, tm * kBM, tn * BN, w.chunk);
              bulk_commit_group();
            }
            continue;
          }
        }
        if (gi < args.Mk) {
#pragma unroll
          for (int c = 0; c < BN / 16; ++c)
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const int gj = tn * BN + c * 16 + t;
              if (gj < args.Nk &&
                  HEAL_DCHECK(((long long)w.chunk * args.Nk + gj) * args.Mk + gi < args.ws_elems, args.status, 151))
                wsc[(size_t)gj * args.Mk + gi] = __uint_as_float(r[c][t]);
            }
        }
        continue;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
      if (!args.splitk && w.chunk == w.nc - 1 && gi < args.Mk) {
        // store the finished row slice of C
        const int gj0 = tn * BN;
        if (args.out_sj == 1) {
          float* orow = args.out + (size_t)gi * args.out_si + gj0;
          const bool vec = ((reinterpret_cast<uintptr_t>(orow) & 15) == 0) && (gj0 + BN <= args.Nk);
          if (vec) {
#pragma unroll
            for (int t = 0; t < BN; t += 4)
              if (HEAL_DCHECK((long long)gi * args.out_si + gj0 + t + 3 < args.out_extent, args.status, 152))
                *reinterpret_cast<float4*>(orow + t) = make_float4(acc[t], acc[t + 1], acc[t + 2], acc[t + 3]);
          } else {
#pragma unroll
            for (int t = 0; t < BN; ++t)
              if (gj0 + t < args.Nk &&
                  HEAL_DCHECK((long long)gi * args.out_si + gj0 + t < args.out_extent, args.status, 153))
                orow[t] = acc[t];
          }
        } else {
#pragma unroll
          for (int t = 0; t < BN; ++t)
            if (gj0 + t < args.Nk) {
              const long long o = (long long)gi * args.out_si + (long long)(gj0 + t) * args.out_sj;
              if (HEAL_DCHECK(o < args.out_extent, args.status, 154)) args.out[o] = acc[t];
            }
        }
      }
    }
    if constexpr (C::kStoreBytes > 0 && B_PRE == 0) {
      if (args.ws_tma && warp == kEpiWarp0 && lane == 0) bulk_wait_group0();   // every tile stored
    }
    (void)ok;
  }

  tc_fence_before();
  __syncthreads();
  // chain mode: no CTA leaves while a peer may still write into its shared memory
  if (args.chain) cluster_sync_all();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, (uint32_t)args.tmem_cols);
}

// ---------------------------------------------------------------------------------
// CTA-pair kernel (cluster of 2, tcgen05 cta_group::2): one 256 x 256 tile of C per pair.
// Each CTA stages its own 128 rows of A and its own 128 columns of B (64 KB per stage,
// three stages) and splits them in place, exactly as the single-CTA kernel does; the
// leader's MMA thread issues M=256, N=256 MMAs that read both CTAs' shared memory, and
// each CTA's TMEM receives its 128 rows x 256 columns.  Barriers that the peer must reach
// are addressed through the cluster window (mapa); completions are committed separately
// to each CTA's barrier.  16 warps: 0 TMA, 1 MMA (leader), 2-7 split, 8-15 epilogue
// (two warps per TMEM lane quarter, 128 columns each, 168 registers via setmaxnreg).
// Chunk arithmetic and the ascending FP32 chunk sum are those of heal_gemm_kernel, so C is
// identical bit for bit.
// ---------------------------------------------------------------------------------
constexpr int kPairSplitWarps = 6;
constexpr int kPairEpiWarp0 = 2 + kPairSplitWarps, kPairEpiWarps = 8;
constexpr int kPairThreads = (kPairEpiWarp0 + kPairEpiWarps) * 32;
// Register split: the epilogue keeps 128 FP32 sums per thread (168 registers); the other
// warps give theirs back.  setmaxnreg.inc draws on the registers the block was launched
// with, so the shares must add up to no more than threads x the compiled register count;
// the host checks that count before the first launch (eight split warps, for instance,
// compile to 96 registers per thread, too few for this split).
constexpr int kPairEpiRegs = 168;
constexpr int kPairLaunchRegs = (65536 / kPairThreads) / 8 * 8;
constexpr int kPairOtherRegs =
    ((kPairLaunchRegs * kPairThreads - kPairEpiRegs * kPairEpiWarps * 32) / (kPairEpiWarp0 * 32)) / 8 * 8 > 88
        ? 88
        : ((kPairLaunchRegs * kPairThreads - kPairEpiRegs * kPairEpiWarps * 32) / (kPairEpiWarp0 * 32)) / 8 * 8;
static_assert(kPairEpiWarp0 * 32 * kPairOtherRegs + kPairEpiWarps * 32 * kPairEpiRegs <= kPairLaunchRegs * kPairThreads,
              "register shares exceed the launch allocation");
// Region pairs of a stage handed to split warp sw: the contiguous run [first, first + count)
// of the n pairs (n = 32: A and B split here; n = 16: only A).  The shares follow the SM
// sub-partitions: split warps sw = 2, 3 (warps 4, 5) are the only split warps on theirs,
// beside the producer (warp 0) and the MMA issuer or forwarder (warp 1), which mostly wait;
// the other four share theirs two by two, so the two lone warps take the larger shares.
// (first, count) of every warp is packed 10 bits per warp (6 + 4): register arithmetic
// rather than a table in local memory.
constexpr uint64_t pack_shares(int s0, int s1, int s2, int s3, int s4, int s5) {
  const int c[6] = {s0, s1, s2, s3, s4, s5};
  uint64_t v = 0;
  int first = 0;
  for (int i = 0; i < 6; ++i) {
    v |= (uint64_t)(first | (c[i] << 6)) << (10 * i);
    first += c[i];
  }
  return v;
}
__device__ __forceinline__ void split_share(int sw, int n, int& first, int& count) {
  //                                      sw: 0  1  2  3  4  5
  constexpr uint64_t k32 = pack_shares(5, 5, 6, 6, 5, 5), k16 = pack_shares(3, 3, 3, 3, 2, 2);
  const uint32_t e = (uint32_t)((n == 32 ? k32 : k16) >> (10 * sw)) & 1023u;
  first = (int)(e & 63u);
  count = (int)(e >> 6);
}
static_assert(kPairSplitWarps == 6, "split_share's tables are written for six split warps");
constexpr int kPairRows = 128;                      // rows of A and of B per CTA
constexpr int kPairN = 256;                         // MMA N (= B columns per pair)
constexpr int kPairStageBytes = 2 * kPairRows * kBK * 4;
constexpr int kPairStages = 3;
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + 1024 + 1024;

template <bool B_MN, int FMT, int B_PRE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    heal_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmB_lo, const GemmArgs args) {
  constexpr int S = kPairStages;
  constexpr int kLoShift = FMT == 0 ? 11 : 0;
  constexpr uint32_t kIdesc = idesc_f16(256, kPairN, FMT, 0, B_MN ? 1 : 0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * kPairStageBytes);
  uint64_t* full = bars;                   // TMA -> split (local)
  uint64_t* split_done = bars + S;         // split warps of both CTAs -> leader's MMA thread
  uint64_t* empty = bars + 2 * S;          // MMA commit -> TMA (both CTAs)
  uint64_t* acc_full = bars + 3 * S;       // MMA commit -> epilogue (both CTAs)
  uint64_t* acc_empty = bars + 3 * S + 2;  // epilogue warps of both CTAs -> leader
  uint64_t* mma_done = bars + 3 * S + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 3 * S + 6);
  uint64_t* split_local = bars + 3 * S + 8;  // peer CTA: its split warps -> its forwarder thread
  uint64_t* acc_local = bars + 4 * S + 8;    // peer CTA: its epilogue warps -> its forwarder thread

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int ntiles = args.tiles_m * args.tiles_n, nc = args.num_chunks;

  pdl_launch_dependents();   // a following kernel may be scheduled; it waits for this grid
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&split_done[s], kPairSplitWarps + 1);   // the leader's split warps + the peer's forwarder
      mbar_init(&split_local[s], kPairSplitWarps);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kPairEpiWarps + 1);   // the leader's epilogue warps + the peer's forwarder
      mbar_init(&acc_local[b], kPairEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    setmaxnreg_dec<kPairOtherRegs>();
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (B_PRE == 1) tma_prefetch_desc(&tmB_lo);
      pdl_wait_prerequisites();   // the operands may come from the preceding kernel
      // A's row tiles are read again for every column stripe of their group: keep them in
      // L2 ahead of B's stripes (5% fewer DRAM reads at 4096 x 14336 x 4096)
      const uint64_t pol_a = l2_policy_evict_last();
      int it = 0;
      bool ok = true;
      for (int tile = cid; tile < ntiles && ok; tile += ncl) {
        int tm, tn;
        tile_coords(tile, args.tiles_m, args.tiles_n, tm, tn);
        for (int ch = 0; ch < nc; ++ch, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag, args.status, 300)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + s * kPairStageBytes;
          mbar_arrive_expect_tx(&full[s], kPairStageBytes - (B_PRE == 2 ? kPairRows * kBK * 2 : 0));
          load_operand_once<kPairRows, false, 0>(st, &tmA, &tmA, &full[s], tm * 256 + kPairRows * (int)rank, ch * kBK,
                                                 pol_a);
          load_operand<kPairRows, B_MN, B_PRE>(st + kPairRows * kBK * 4, &tmB, &tmB_lo, &full[s],
                                               tn * kPairN + kPairRows * (int)rank, ch * kBK);
        }
      }
      for (int j = 0; j < S && j < it; ++j) {
        const int jt = it - 1 - j;
        volatile int dummy = 0;
        mbar_wait(&full[jt % S], (uint32_t)(jt / S) & 1u, &dummy, args.status, 301);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader CTA) ------------------------------
    setmaxnreg_dec<kPairOtherRegs>();
    if (rank == 0 && lane == 0) {
      const uint32_t peer = 1u;
      int it = 0;
      bool ok = true;
      for (int tile = cid; tile < ntiles && ok; tile += ncl) {
        for (int ch = 0; ch < nc; ++ch, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          const int b = it & 1;
          const uint32_t aph = (uint32_t)(it >> 1) & 1u;
          if (!mbar_wait_cluster(&split_done[s], ph, abort_flag, args.status, 310) ||
              !mbar_wait_cluster(&acc_empty[b], aph ^ 1u, abort_flag, args.status, 311)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + s * kPairStageBytes);
          const uint32_t sb = sa + kPairRows * kBK * 4;
          const uint64_t a_hi = OperandDesc<kPairRows, false>::hi(sa), a_lo = OperandDesc<kPairRows, false>::lo(sa);
          const uint64_t b_hi = OperandDesc<kPairRows, B_MN>::hi(sb), b_lo = OperandDesc<kPairRows, B_MN>::lo(sb);
          constexpr uint64_t dA = OperandDesc<kPairRows, false>::kStep, dB = OperandDesc<kPairRows, B_MN>::kStep;
          const uint32_t d = tmem_base + (uint32_t)(b * kPairN);
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j) {
            if constexpr (B_PRE != 2) {
              mma_f16_pair(d, a_hi + j * dA, b_lo + j * dB, kIdesc, j > 0 ? 1u : 0u);
              mma_f16_pair(d, a_lo + j * dA, b_hi + j * dB, kIdesc, 1u);
            } else {
              mma_f16_pair(d, a_lo + j * dA, b_hi + j * dB, kIdesc, j > 0 ? 1u : 0u);
            }
          }
          mma_f16_pair_scale_d<kLoShift>(d, a_hi, b_hi, kIdesc);
#pragma unroll
          for (int j = 1; j < kBK / 16; ++j) mma_f16_pair(d, a_hi + j * dA, b_hi + j * dB, kIdesc, 1u);
          const uint32_t e_loc = smem_u32(&empty[s]), f_loc = smem_u32(&acc_full[b]);
          tc_commit_pair(mapa_shared(e_loc, 0u));
          tc_commit_pair(mapa_shared(e_loc, peer));
          tc_commit_pair(mapa_shared(f_loc, 0u));
          tc_commit_pair(mapa_shared(f_loc, peer));
        }
      }
      tc_commit_pair(mapa_shared(smem_u32(mma_done), 0u));
      volatile int dummy = 0;
      mbar_wait(mma_done, 0, &dummy, args.status, 312);
    } else if (rank == 1 && lane == 0) {
      // ---- forwarder (peer CTA): each stage split here and each chunk drained here becomes
      // one arrive on the leader's split_done / acc_empty.  The two streams interleave in an
      // order that depends on timing, so both are polled.
      const uint32_t sd_leader0 = mapa_shared(smem_u32(&split_done[0]), 0u);
      const uint32_t ae_leader0 = mapa_shared(smem_u32(&acc_empty[0]), 0u);
      const int total = ((ntiles - cid + ncl - 1) / ncl) * nc;   // (tile, chunk) iterations of this pair
      int is = 0, ia = 0;
      uint64_t t0 = globaltimer();
      while ((is < total || ia < total) && !*abort_flag) {
        bool moved = false;
        if (is < total && mbar_test_wait(&split_local[is % S], (uint32_t)(is / S) & 1u)) {
          // release at CTA scope (mbarrier.arrive's default): this thread's acquire of the
          // six local arrivals, each after its warp's split stores into this CTA's shared
          // memory and fence.proxy.async, is ordered before the arrive the leader's MMA thread
          // acquires.  A cluster-scope release costs ~1000 cycles here, CTA scope ~20.
          mbar_arrive_remote(sd_leader0 + (uint32_t)((is % S) * 8));
          ++is;
          moved = true;
        }
        if (ia < total && ia < is && mbar_test_wait(&acc_local[ia & 1], (uint32_t)(ia >> 1) & 1u)) {
          // TMEM reuse only (the drains' tcgen05.ld completed before their tcgen05 fence and
          // arrive; the MMA thread fences after its wait): no data to publish, no release
          mbar_arrive_cluster_relaxed(ae_leader0 + (uint32_t)((ia & 1) * 8));
          ++ia;
          moved = true;
        }
        if (moved) {
          t0 = globaltimer();
        } else {
          __nanosleep(32);   // leave the issue slots to the split and epilogue warps of this sub-partition
          if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            report_timeout(args.status, 313);
          }
        }
      }
    }
  } else if (warp < kPairEpiWarp0) {
    // ------------------------------ split warps (both CTAs) ------------------------------
    setmaxnreg_dec<kPairOtherRegs>();
    pdl_wait_prerequisites();   // chan_exp may come from the preceding kernel
    const int sw = warp - 2;
    constexpr int kPairsA = kPairRows / 8, kPairsB = kPairRows / 8;
    static_assert(kPairEpiWarp0 == 2 + kPairSplitWarps, "split warps are warps 2 .. kPairEpiWarp0 - 1");
    int it = 0;
    bool ok = true;
    for (int tile = cid; tile < ntiles && ok; tile += ncl) {
      for (int ch = 0; ch < nc; ++ch, ++it) {
        const int s = it % S;
        const uint32_t ph = (uint32_t)(it / S) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, args.status, 320)) {
          ok = false;
          break;
        }
        uint8_t* st = stages + s * kPairStageBytes;
        const int k0 = ch * kBK;
        constexpr int kLast = B_PRE ? kPairsA : kPairsA + kPairsB;
        int t0, tn;
        split_share(sw, kLast, t0, tn);
        for (int t = t0; t < t0 + tn; ++t) {
          uint8_t *s0, *s1;
          int kboff;
          if (t < kPairsA) {
            pair_addr<kPairRows, false>(st, t, s0, s1, kboff);
            split_pair<FMT, false>(s0, s1, lane, args.chan_exp, args.expA_sign, k0 + kboff, args.K);
          } else {
            pair_addr<kPairRows, B_MN>(st + kPairRows * kBK * 4, t - kPairsA, s0, s1, kboff);
            split_pair<FMT, B_MN>(s0, s1, lane, args.chan_exp, args.expB_sign, k0 + kboff, args.K);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        // every split warp arrives on a barrier of its own CTA (a CTA-scope release): in the
        // leader on split_done, which its MMA thread waits for; in the peer on split_local,
        // which one thread forwards to the leader (fewer arrivals crossing the cluster than
        // six remote ones per stage, and measured ~2% faster)
        if (lane == 0) mbar_arrive(rank == 0 ? &split_done[s] : &split_local[s]);
      }
    }
  } else {
    // ------------------------------ epilogue (both CTAs) ------------------------------
    setmaxnreg_inc<kPairEpiRegs>();
    pdl_wait_prerequisites();   // C may still be read by the preceding kernel
    const int quarter = warp & 3;
    const int half = (warp - kPairEpiWarp0) >> 2;
    const int i_local = quarter * 32 + lane;
    float acc[128];
#pragma unroll
    for (int t = 0; t < 128; ++t) acc[t] = 0.0f;
    int it = 0;
    bool ok = true;
    for (int tile = cid; tile < ntiles && ok; tile += ncl) {
      int tm, tn;
      tile_coords(tile, args.tiles_m, args.tiles_n, tm, tn);
      const int gi = tm * 256 + kPairRows * (int)rank + i_local;
      for (int ch = 0; ch < nc; ++ch, ++it) {
        const int b = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait_cluster(&acc_full[b], aph, abort_flag, args.status, 330)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * kPairN + half * 128);
        const bool first = (ch == 0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t r[16];
          tmem_ld16(taddr + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float dv = __uint_as_float(r[t]);
            acc[c * 16 + t] = first ? dv : __fadd_rn(acc[c * 16 + t], dv);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(rank == 0 ? &acc_empty[b] : &acc_local[b]);   // see the split warps
      }
      if (!ok) break;
      if (gi < args.Mk) {
        const int gj0 = tn * kPairN + half * 128;
        float* orow = args.out + (size_t)gi * args.out_si + gj0;
        if (((reinterpret_cast<uintptr_t>(orow) & 15) == 0) && (gj0 + 128 <= args.Nk)) {
#pragma unroll
          for (int t = 0; t < 128; t += 4)
            if (HEAL_DCHECK((long long)gi * args.out_si + gj0 + t + 3 < args.out_extent, args.status, 350))
              *reinterpret_cast<float4*>(orow + t) = make_float4(acc[t], acc[t + 1], acc[t + 2], acc[t + 3]);
        } else {
#pragma unroll
          for (int t = 0; t < 128; ++t)
            if (gj0 + t < args.Nk &&
                HEAL_DCHECK((long long)gi * args.out_si + gj0 + t < args.out_extent, args.status, 351))
              orow[t] = acc[t];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 0) tmem_dealloc_pair(tmem_base, 512);
}

// Ordered sum of chunk values: out(i, j) = ((ws[0] + ws[1]) + ws[2]) + ...
// One warp per block and 32 consecutive outputs per warp (lane = output, so every chunk
// row the warp reads is one coalesced 128-byte line).  Each lane requests kRedBatch chunk
// values at once (registers), then adds them in ascending chunk order: K = 4096 takes one
// memory round trip.  Blocks of one warp spread the loads over every SM, and without shared
// memory they fit beside a resident GEMM CTA: launched with programmatic dependent launch
// they are already on the SMs, waiting, when the GEMM grid finishes.
constexpr int kRedBatch = 64;
__global__ void __launch_bounds__(32) heal_chunk_reduce_kernel(const float* __restrict__ ws, int num_chunks, int Mk,
                                                               int Nk, float* out, long long si, long long sj,
                                                               long long out_extent, unsigned int* status) {
  pdl_launch_dependents();   // the next kernel may be scheduled; it waits for this grid
  pdl_wait_prerequisites();   // the GEMM kernel that wrote ws has completed
  const long long o = (long long)blockIdx.x * 32 + threadIdx.x;
  if (o >= (long long)Mk * Nk) return;
  const int i = (int)(o % Mk), j = (int)(o / Mk);
  const size_t plane = (size_t)Mk * Nk;
  const float* p = ws + (size_t)j * Mk + i;
  float acc = 0.0f;
  for (int c0 = 0; c0 < num_chunks; c0 += kRedBatch) {
    const int cn = min(kRedBatch, num_chunks - c0);
    float v[kRedBatch];
#pragma unroll
    for (int t = 0; t < kRedBatch; ++t) v[t] = t < cn ? __ldcs(p + (size_t)(c0 + t) * plane) : 0.0f;
    // every value is requested before the first add (the loads must not be interleaved with
    // the dependent adds, which would make one memory round trip per chunk)
#pragma unroll
    for (int t = 0; t < kRedBatch; ++t) asm volatile("" ::"f"(v[t]));
#pragma unroll
    for (int t = 0; t < kRedBatch; ++t)
      if (t < cn) acc = (c0 + t == 0) ? v[t] : __fadd_rn(acc, v[t]);
  }
  const long long oi = (long long)i * si + (long long)j * sj;
  if (HEAL_DCHECK(oi < out_extent, status, 160)) out[oi] = acc;
}

// The same ordered sum for large outputs (M >= 32: 8-67 MB of chunk values): each lane
// takes four consecutive outputs of one column j and reads them as one 16-byte vector per
// chunk, so a warp moves 512 contiguous bytes of each chunk plane per request (4x longer
// runs in DRAM than the one-value-per-lane kernel), kRedWideBatch chunks per round trip.
constexpr int kRedWideBatch = 16;
__global__ void __launch_bounds__(128) heal_chunk_reduce_wide_kernel(const float* __restrict__ ws, int num_chunks,
                                                                     int Mk, int Nk, float* out, long long sj,
                                                                     long long out_extent, unsigned int* status) {
  pdl_launch_dependents();   // the next kernel may be scheduled; it waits for this grid
  pdl_wait_prerequisites();   // the GEMM kernel that wrote ws has completed
  const int q4 = Mk / 4;     // float4 per column (Mk % 4 == 0)
  const long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // float4 index
  if (v >= (long long)q4 * Nk) return;
  const int j = (int)(v / q4), i0 = (int)(v % q4) * 4;
  const size_t plane4 = (size_t)Mk * Nk / 4;
  const float4* p = reinterpret_cast<const float4*>(ws) + (size_t)j * q4 + i0 / 4;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int c0 = 0; c0 < num_chunks; c0 += kRedWideBatch) {
    const int cn = min(kRedWideBatch, num_chunks - c0);
    float4 x[kRedWideBatch];
#pragma unroll
    for (int t = 0; t < kRedWideBatch; ++t)
      x[t] = t < cn ? __ldcs(p + (size_t)(c0 + t) * plane4) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    // all requested before the first add (not sunk into the dependent adds)
#pragma unroll
    for (int t = 0; t < kRedWideBatch; ++t) asm volatile("" ::"f"(x[t].x), "f"(x[t].y), "f"(x[t].z), "f"(x[t].w));
#pragma unroll
    for (int t = 0; t < kRedWideBatch; ++t) {
      if (t >= cn) break;
      const bool first = (c0 + t == 0);
      acc[0] = first ? x[t].x : __fadd_rn(acc[0], x[t].x);
      acc[1] = first ? x[t].y : __fadd_rn(acc[1], x[t].y);
      acc[2] = first ? x[t].z : __fadd_rn(acc[2], x[t].z);
      acc[3] = first ? x[t].w : __fadd_rn(acc[3], x[t].w);
    }
  }
  // out(i, j) at out[i + j * sj]
  float* o = out + (long long)j * sj + i0;
  if (HEAL_DCHECK((long long)j * sj + i0 + 3 < out_extent, status, 161)) {
    if ((reinterpret_cast<uintptr_t>(o) & 15) == 0)
      *reinterpret_cast<float4*>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    else {
      o[0] = acc[0];
      o[1] = acc[1];
      o[2] = acc[2];
      o[3] = acc[3];
    }
  }
}

// ---------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------
namespace {

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_elems * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return encode_tensor_map(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

// Operand tensor map: R rows of the tile, matrix with `rows` rows and K columns where
// element (row, k) lives at base[row*ld + k] (K-major) or base[k*ld + row] (MN-major).
bool operand_map(CUtensorMap* map, const void* base, bool mn, bool is16, int rows, int K, long long ld, int R) {
  const CUtensorMapDataType dt = is16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const int eb = is16 ? 2 : 4;
  const uint32_t inner_box = is16 ? 64u : 32u;   // 128 bytes
  if (!mn) return encode_2d(map, dt, eb, base, (uint64_t)K, (uint64_t)rows, (uint64_t)ld, inner_box, (uint32_t)R);
  return encode_2d(map, dt, eb, base, (uint64_t)rows, (uint64_t)K, (uint64_t)ld, inner_box, 64u);
}

template <int BN, bool A_MN, bool B_MN, int FMT, bool CORR_SWAP, int A_PRE, int B_PRE>
cudaError_t launch_variant(const CUtensorMap& a, const CUtensorMap& alo, const CUtensorMap& b,
                           const CUtensorMap& blo, const GemmArgs& args, int grid, cudaStream_t stream) {
  auto kern = heal_gemm_kernel<BN, A_MN, B_MN, FMT, CORR_SWAP, A_PRE, B_PRE>;
  const int smem = Cfg<BN>::kSmemBytes;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    if (BN == 128) {
      // setmaxnreg shares (8 warps at 96, 4 epilogue warps at 240) must fit the launch allocation
      cudaFuncAttributes fa{};
      e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      if ((long long)fa.numRegs * Roles<BN>::kThreads < 8LL * 32 * 96 + 4LL * 32 * 240) return cudaErrorInvalidConfiguration;
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  // programmatic dependent launch: the grid may start during the preceding kernel; every
  // role waits for it (griddepcontrol.wait) before touching data it may produce or read
  if (args.chain)
    return launch_pdl_cluster(kern, dim3(grid), dim3(Roles<BN>::kThreads), (size_t)smem, stream, args.chain, a, alo,
                              b, blo, args);
  return launch_pdl(kern, dim3(grid), dim3(Roles<BN>::kThreads), (size_t)smem, stream, a, alo, b, blo, args);
}

template <int BN, bool A_MN, bool B_MN, bool CORR_SWAP, int A_PRE, int B_PRE>
cudaError_t launch_fmt(int fmt, const CUtensorMap& a, const CUtensorMap& alo, const CUtensorMap& b,
                       const CUtensorMap& blo, const GemmArgs& args, int grid, cudaStream_t stream) {
  if (fmt == 0) return launch_variant<BN, A_MN, B_MN, 0, CORR_SWAP, A_PRE, B_PRE>(a, alo, b, blo, args, grid, stream);
  return launch_variant<BN, A_MN, B_MN, 1, CORR_SWAP, A_PRE, B_PRE>(a, alo, b, blo, args, grid, stream);
}

// Swapped-operand skinny kernels: kernel-A = the weights (pre-split or FP32), kernel-B =
// the M <= 64 activation rows padded to BN = 16 / 32 / 64.
template <int PRE>
cudaError_t launch_skinny(int BNk, bool b_mn, int fmt, const CUtensorMap& a, const CUtensorMap& alo,
                          const CUtensorMap& b, const CUtensorMap& blo, const GemmArgs& args, int grid,
                          cudaStream_t stream) {
  if (BNk == 16)
    return b_mn ? launch_fmt<16, true, false, true, PRE, 0>(fmt, a, alo, b, blo, args, grid, stream)
                : launch_fmt<16, false, false, true, PRE, 0>(fmt, a, alo, b, blo, args, grid, stream);
  if (BNk == 32)
    return b_mn ? launch_fmt<32, true, false, true, PRE, 0>(fmt, a, alo, b, blo, args, grid, stream)
                : launch_fmt<32, false, false, true, PRE, 0>(fmt, a, alo, b, blo, args, grid, stream);
  return b_mn ? launch_fmt<64, true, false, true, PRE, 0>(fmt, a, alo, b, blo, args, grid, stream)
              : launch_fmt<64, false, false, true, PRE, 0>(fmt, a, alo, b, blo, args, grid, stream);
}

template <bool B_MN, int FMT, int B_PRE>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& blo, const GemmArgs& args,
                        int grid, cudaStream_t stream) {
  auto kern = heal_gemm_pair_kernel<B_MN, FMT, B_PRE>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    // the warps' register shares must fit the registers the block is launched with
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if ((long long)fa.numRegs * kPairThreads <
        (long long)kPairEpiWarp0 * 32 * kPairOtherRegs + (long long)kPairEpiWarps * 32 * kPairEpiRegs)
      return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(kPairThreads), (size_t)kPairSmemBytes, stream, a, b, blo, args);
}

template <int PRE>
cudaError_t launch_pair_fmt(bool b_mn, int fmt, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& blo,
                            const GemmArgs& args, int grid, cudaStream_t stream) {
  if (fmt == 0)
    return b_mn ? launch_pair<true, 0, PRE>(a, b, blo, args, grid, stream)
                : launch_pair<false, 0, PRE>(a, b, blo, args, grid, stream);
  return b_mn ? launch_pair<true, 1, PRE>(a, b, blo, args, grid, stream)
              : launch_pair<false, 1, PRE>(a, b, blo, args, grid, stream);
}

// 128 x 128 tiles in the caller's operand order
template <int PRE>
cudaError_t launch_wide(bool b_mn, int fmt, const CUtensorMap& a, const CUtensorMap& alo, const CUtensorMap& b,
                        const CUtensorMap& blo, const GemmArgs& args, int grid, cudaStream_t stream) {
  return b_mn ? launch_fmt<128, false, true, false, 0, PRE>(fmt, a, alo, b, blo, args, grid, stream)
              : launch_fmt<128, false, false, false, 0, PRE>(fmt, a, alo, b, blo, args, grid, stream);
}

}  // namespace

// CTAs per tile in chain mode: as many as the SMs allow for one wave of tiles (at most 8,
// the portable cluster size, and at most one per chunk), provided each CTA's chunks fit in
// TMEM as separate accumulators; 0 when no chain of at least two CTAs fits.
int chain_size(int tiles, int nc, int BNk, int sms) {
  if (BNk > 32 || tiles <= 0) return 0;
  int S = sms / tiles;
  if (S > 8) S = 8;
  if (S > nc) S = nc;
  if (S < 2) return 0;
  if ((long long)((nc + S - 1) / S) * BNk > 512) return 0;
  return S;
}

size_t gemm_workspace_bytes(int M, int N, int K, int tile_config) {
  if (tile_config != HEAL_TILE_SKINNY_SPLITK) return 0;
  const size_t nc = (size_t)((K + kBK - 1) / kBK);
  const size_t mpad = (size_t)(M <= 16 ? 16 : M <= 32 ? 32 : 64);
  (void)mpad;
  return nc * (size_t)M * (size_t)N * sizeof(float);
}

heal_status_t gemm_launch(int M, int N, int K, const float* A, long long lda, const void* B, long long ldb,
                          float* Cout, long long ldc, int fmt, const heal_gemm_opts_t& o, cudaStream_t stream) {
  int cfg = o.tile_config;
  const int sms = device_sm_count();
  if (sms <= 0) return HEAL_ERR_CUDA;
  if (cfg == HEAL_TILE_AUTO) {
    const int bnk = M <= 16 ? 16 : 32;
    if (M <= 64 && o.workspace != nullptr && o.workspace_bytes >= gemm_workspace_bytes(M, N, K, HEAL_TILE_SKINNY_SPLITK))
      cfg = HEAL_TILE_SKINNY_SPLITK;
    else if (M <= 32 && chain_size((N + kBM - 1) / kBM, (K + kBK - 1) / kBK, bnk, sms) >= 2)
      cfg = HEAL_TILE_SKINNY_CHAIN;   // no workspace: K still spread over the SMs
    else if (M >= 256 && N >= 256)
      cfg = HEAL_TILE_256x256_PAIR;
    else
      cfg = HEAL_TILE_128x128;
  }
  const bool b_mn = (o.b_layout == 0);   // B stored K x N: N contiguous
  const int nc = (K + kBK - 1) / kBK;
  CUtensorMap ta{}, talo{}, tb{}, tblo{};
  GemmArgs args{};
  args.K = K;
  args.num_chunks = nc;
  args.chan_exp = o.chan_exp;
  args.static_op = 0;
  const int pre = o.b_presplit;   // 0 FP32 B, 1 pre-split hi + lo, 2 16-bit B (two products)
  args.status = device_status_ptr();
  args.out_extent = (long long)(M - 1) * ldc + N;   // C is M x N with row stride ldc in every config
  args.ws_elems = o.workspace ? (long long)(o.workspace_bytes / sizeof(float)) : 0;
  cudaError_t err = cudaSuccess;

  if (cfg == HEAL_TILE_256x256_PAIR) {
    args.Mk = M;
    args.Nk = N;
    args.tiles_m = (M + 255) / 256;
    args.tiles_n = (N + 255) / 256;
    args.splitk = 0;
    args.out = Cout;
    args.out_si = ldc;
    args.out_sj = 1;
    args.expA_sign = -1;
    args.expB_sign = +1;
    if (!operand_map(&ta, A, false, false, M, K, lda, kPairRows)) return HEAL_ERR_CUDA;
    if (!operand_map(&tb, B, b_mn, pre != 0, N, K, ldb, kPairRows)) return HEAL_ERR_CUDA;
    if (pre == 1 && !operand_map(&tblo, o.b_lo, b_mn, true, N, K, ldb, kPairRows)) return HEAL_ERR_CUDA;
    const long long pairs = (long long)args.tiles_m * args.tiles_n;
    const int max_pairs = sms / 2;
    const int grid = 2 * (int)(pairs < max_pairs ? pairs : max_pairs);
    if (grid < 2) return HEAL_ERR_CUDA;
    err = pre == 0 ? launch_pair_fmt<0>(b_mn, fmt, ta, tb, tblo, args, grid, stream)
        : pre == 1 ? launch_pair_fmt<1>(b_mn, fmt, ta, tb, tblo, args, grid, stream)
                   : launch_pair_fmt<2>(b_mn, fmt, ta, tb, tblo, args, grid, stream);
    return err == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
  }

  if (cfg == HEAL_TILE_128x128) {
    constexpr int BN = 128;
    args.Mk = M;
    args.Nk = N;
    args.tiles_m = (M + kBM - 1) / kBM;
    args.tiles_n = (N + BN - 1) / BN;
    args.splitk = 0;
    args.out = Cout;
    args.out_si = ldc;
    args.out_sj = 1;
    args.expA_sign = -1;
    args.expB_sign = +1;
    args.static_op = o.b_static ? 2 : 0;   // kernel-B = B
    args.tmem_cols = Cfg<BN>::kTmemCols;
    if (!operand_map(&ta, A, false, false, M, K, lda, kBM)) return HEAL_ERR_CUDA;
    if (!operand_map(&tb, B, b_mn, pre != 0, N, K, ldb, BN)) return HEAL_ERR_CUDA;
    if (pre == 1 && !operand_map(&tblo, o.b_lo, b_mn, true, N, K, ldb, BN)) return HEAL_ERR_CUDA;
    const int ntiles = args.tiles_m * args.tiles_n;
    const int grid = ntiles < sms ? ntiles : sms;
    err = pre == 0 ? launch_wide<0>(b_mn, fmt, ta, talo, tb, tblo, args, grid, stream)
        : pre == 1 ? launch_wide<1>(b_mn, fmt, ta, talo, tb, tblo, args, grid, stream)
                   : launch_wide<2>(b_mn, fmt, ta, talo, tb, tblo, args, grid, stream);
    return err == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
  }

  if (cfg == HEAL_TILE_SKINNY_SPLITK || cfg == HEAL_TILE_SKINNY_FULLK || cfg == HEAL_TILE_SKINNY_CHAIN) {
    const bool split = (cfg == HEAL_TILE_SKINNY_SPLITK);
    if (M > 64) return HEAL_ERR_UNSUPPORTED;
    if (split && (o.workspace == nullptr || o.workspace_bytes < gemm_workspace_bytes(M, N, K, cfg)))
      return HEAL_ERR_INVALID_ARGUMENT;
    // swapped roles: kernel-A = B^T (N rows), kernel-B = A (M rows), C written transposed
    args.Mk = N;
    args.Nk = M;
    args.tiles_m = (N + kBM - 1) / kBM;
    args.tiles_n = 1;
    args.splitk = split ? 1 : 0;
    args.ws = static_cast<float*>(o.workspace);
    args.out = Cout;
    args.out_si = 1;
    args.out_sj = ldc;
    args.expA_sign = +1;
    args.expB_sign = -1;
    args.static_op = o.b_static ? 1 : 0;   // kernel-A = B^T
    const int BNk = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    args.tmem_cols = 4 * BNk < 32 ? 32 : 4 * BNk;   // four accumulator buffers (Cfg::kAccBufs)
    args.chain = 0;
    const int S = cfg == HEAL_TILE_SKINNY_CHAIN ? chain_size(args.tiles_m, nc, BNk, sms) : 0;
    if (S >= 2) {
      args.chain = S;
      const int per = (nc + S - 1) / S;
      int cols = 32;
      while (cols < per * BNk) cols *= 2;
      args.tmem_cols = cols;
    }
    if (!operand_map(&ta, B, b_mn, pre != 0, N, K, ldb, kBM)) return HEAL_ERR_CUDA;
    if (pre == 1 && !operand_map(&talo, o.b_lo, b_mn, true, N, K, ldb, kBM)) return HEAL_ERR_CUDA;
    if (!operand_map(&tb, A, false, false, M, K, lda, BNk)) return HEAL_ERR_CUDA;
    args.ws_tma = 0;
    if (split && BNk == 64 && N % 4 == 0 && (reinterpret_cast<uintptr_t>(o.workspace) & 15) == 0) {
      // the workspace as [nc][M][N] FP32 for the TMA stores of chunk tiles (BN x 128)
      const cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)nc};
      const cuuint64_t strides[2] = {(cuuint64_t)N * 4, (cuuint64_t)N * M * 4};
      const cuuint32_t box[3] = {(cuuint32_t)kBM, 64u, 1u};
      const cuuint32_t es[3] = {1, 1, 1};
      if (!encode_tensor_map(&tblo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, o.workspace, dims, strides, box, es,
                             CU_TENSOR_MAP_SWIZZLE_NONE))
        return HEAL_ERR_CUDA;
      args.ws_tma = 1;
    }
    const long long units = split ? (long long)args.tiles_m * nc : (long long)args.tiles_m;
    const int grid = args.chain ? args.tiles_m * args.chain : (int)(units < sms ? units : sms);
    err = pre == 0 ? launch_skinny<0>(BNk, b_mn, fmt, ta, talo, tb, tblo, args, grid, stream)
        : pre == 1 ? launch_skinny<1>(BNk, b_mn, fmt, ta, talo, tb, tblo, args, grid, stream)
                   : launch_skinny<2>(BNk, b_mn, fmt, ta, talo, tb, tblo, args, grid, stream);
    if (err != cudaSuccess) return HEAL_ERR_CUDA;
    if (!split) return HEAL_OK;
    if (M >= 32 && N % 4 == 0 && (reinterpret_cast<uintptr_t>(o.workspace) & 15) == 0) {
      const long long vec = (long long)N / 4 * M;
      const long long wblocks = (vec + 127) / 128;
      if (wblocks >= (1LL << 31)) return HEAL_ERR_UNSUPPORTED;
      const cudaError_t e = launch_pdl(heal_chunk_reduce_wide_kernel, dim3((unsigned)wblocks), dim3(128), 0, stream,
                                       (const float*)args.ws, nc, N, M, Cout, (long long)ldc, args.out_extent,
                                       args.status);
      return e == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
    }
    const long long rblocks = ((long long)N * M + 31) / 32;
    if (rblocks >= (1LL << 31)) return HEAL_ERR_UNSUPPORTED;
    const cudaError_t e = launch_pdl(heal_chunk_reduce_kernel, dim3((unsigned)rblocks), dim3(32), 0, stream,
                                     (const float*)args.ws, nc, N, M, Cout, 1LL, (long long)ldc, args.out_extent,
                                     args.status);
    return e == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
  }
  return HEAL_ERR_UNSUPPORTED;
}

}  // namespace heal
