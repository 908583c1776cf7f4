// heal_api.cu -- the C ABI of libheal.so: host-side validation, dispatch, device status.
// Every check here runs before any launch; a rejected call launches nothing.
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "heal_internal.h"
#include "heal_ptx.cuh"

namespace heal {

__device__ unsigned int g_status[2];

unsigned int* device_status_ptr() {
  static unsigned int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev < 64 && cache[dev]) return cache[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (dev < 64) cache[dev] = static_cast<unsigned int*>(p);
  return static_cast<unsigned int*>(p);
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev < 64) cache[dev] = n;
  return n;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, cuuint32_t rank, void* base, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box, const cuuint32_t* elem_strides,
                       CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const CUresult r = fn(map, dt, rank, base, dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// One warp waits, through the same bounded wait every kernel uses, on an mbarrier that
// nothing arrives on; the wait gives up after limit_ns and records a timeout.
__global__ void heal_wait_probe_kernel(unsigned int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0u, &abort_flag, status, 900, limit_ns);
}

}  // namespace heal

using namespace heal;

extern "C" {

heal_status_t heal_split(const float* x, void* hi, void* lo, int64_t n, heal_split_fmt_t fmt, heal_stream_t stream) {
  if (n < 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (fmt != HEAL_SPLIT_FP16_S11 && fmt != HEAL_SPLIT_BF16) return HEAL_ERR_INVALID_ARGUMENT;
  if (n == 0) return HEAL_OK;
  if (!x || !hi || !lo) return HEAL_ERR_INVALID_ARGUMENT;
  if (!aligned(x, 4) || !aligned(hi, 2) || !aligned(lo, 2)) return HEAL_ERR_INVALID_ARGUMENT;
  const heal_status_t st = split_launch(x, hi, lo, (long long)n, (int)fmt, (cudaStream_t)stream);
  if (st == HEAL_ERR_CUDA) (void)cudaGetLastError();
  return st;
}

// Split-K scratch of the tile configuration (0 when it uses none), rounded up to 256 bytes.
static size_t splitk_bytes(int M, int N, int K, int cfg) {
  const size_t b = cfg == HEAL_TILE_AUTO ? (M <= 64 ? gemm_workspace_bytes(M, N, K, HEAL_TILE_SKINNY_SPLITK) : 0)
                                         : gemm_workspace_bytes(M, N, K, cfg);
  return (b + 255) & ~(size_t)255;
}

size_t heal_gemm_workspace_bytes(int M, int N, int K, const heal_gemm_opts_t* opts) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const int cfg = opts ? opts->tile_config : HEAL_TILE_AUTO;
  const size_t b = splitk_bytes(M, N, K, cfg);
  if (opts && opts->b_split_pass == 1) return b + (size_t)4 * K * N;   // hi and lo parts of B
  if (cfg == HEAL_TILE_AUTO) return M <= 64 ? gemm_workspace_bytes(M, N, K, HEAL_TILE_SKINNY_SPLITK) : 0;
  return gemm_workspace_bytes(M, N, K, cfg);
}

heal_status_t heal_gemm_compensated(int M, int N, int K, const float* A, int64_t lda, const void* B, int64_t ldb,
                                    float* C, int64_t ldc, heal_split_fmt_t fmt, const heal_gemm_opts_t* opts,
                                    heal_stream_t stream) {
  heal_gemm_opts_t o{};
  o.tile_config = HEAL_TILE_AUTO;
  if (opts) o = *opts;
  if (M <= 0 || N <= 0 || K <= 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (!A || !B || !C) return HEAL_ERR_INVALID_ARGUMENT;
  if (fmt != HEAL_SPLIT_FP16_S11 && fmt != HEAL_SPLIT_BF16) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_layout != 0 && o.b_layout != 1) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_presplit < 0 || o.b_presplit > 2) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_static != 0 && o.b_static != 1) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_split_pass != 0 && o.b_split_pass != 1) return HEAL_ERR_INVALID_ARGUMENT;
  for (int r : o.reserved)
    if (r != 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.tile_config < HEAL_TILE_AUTO || o.tile_config > HEAL_TILE_SKINNY_CHAIN) return HEAL_ERR_INVALID_ARGUMENT;
  // TMA: 16-byte aligned bases, row strides multiples of 16 bytes
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 4)) return HEAL_ERR_INVALID_ARGUMENT;
  if (lda < K || lda % 4 != 0) return HEAL_ERR_INVALID_ARGUMENT;
  const int64_t b_min = o.b_layout == 0 ? N : K;
  if (ldb < b_min || ldb % (o.b_presplit ? 8 : 4) != 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (ldc < N) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_presplit == 1 && (!o.b_lo || !aligned(o.b_lo, 16))) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_presplit == 2 && o.b_lo) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.chan_exp && !aligned(o.chan_exp, 1)) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.workspace && !aligned(o.workspace, 16)) return HEAL_ERR_INVALID_ARGUMENT;
  if (o.b_split_pass) {
    // split B into the workspace (after the split-K part), then the product on its parts
    if (o.b_presplit != 0 || o.chan_exp != nullptr) return HEAL_ERR_INVALID_ARGUMENT;
    if (ldb != b_min || ldb % 8 != 0) return HEAL_ERR_UNSUPPORTED;   // 16-byte rows of the 16-bit parts
    const size_t head = splitk_bytes(M, N, K, o.tile_config);
    if (!o.workspace || o.workspace_bytes < head + (size_t)4 * K * N) return HEAL_ERR_INVALID_ARGUMENT;
    uint8_t* w = static_cast<uint8_t*>(o.workspace);
    void* bhi = w + head;
    void* blo = w + head + (size_t)2 * K * N;
    heal_status_t st = split_launch(static_cast<const float*>(B), bhi, blo, (long long)K * N, (int)fmt,
                                    (cudaStream_t)stream);
    if (st == HEAL_OK) {
      heal_gemm_opts_t o2 = o;
      o2.b_split_pass = 0;
      o2.b_presplit = 1;
      o2.b_lo = blo;
      o2.b_static = 0;                 // B's parts are written by the launch just before
      o2.workspace_bytes = head;
      if (head == 0) o2.workspace = nullptr;
      st = gemm_launch(M, N, K, A, lda, bhi, ldb, C, ldc, (int)fmt, o2, (cudaStream_t)stream);
    }
    if (st == HEAL_ERR_CUDA) (void)cudaGetLastError();
    return st;
  }
  const heal_status_t st = gemm_launch(M, N, K, A, lda, B, ldb, C, ldc, (int)fmt, o, (cudaStream_t)stream);
  if (st == HEAL_ERR_CUDA) (void)cudaGetLastError();
  return st;
}

heal_status_t heal_kv_quantize_int16(const void* x, int x_is_bf16, int B, int T, int H, int D, int64_t x_stride_batch,
                                     int64_t x_stride_tok, int64_t x_stride_head, int16_t* q_cache,
                                     float* scale_cache, int Tmax, int t_offset, heal_stream_t stream) {
  if (B < 0 || T < 0 || H < 0 || Tmax < 0 || t_offset < 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (x_is_bf16 != 0 && x_is_bf16 != 1) return HEAL_ERR_INVALID_ARGUMENT;
  if (D < 8 || D > 256 || (D & (D - 1)) != 0) return HEAL_ERR_UNSUPPORTED;
  if ((long long)t_offset + T > Tmax) return HEAL_ERR_INVALID_ARGUMENT;
  if ((long long)B * T * H == 0) return HEAL_OK;
  if (!x || !q_cache || !scale_cache) return HEAL_ERR_INVALID_ARGUMENT;
  if (!aligned(x, 16) || !aligned(q_cache, 16) || !aligned(scale_cache, 4)) return HEAL_ERR_INVALID_ARGUMENT;
  if (x_stride_batch % 8 || x_stride_tok % 8 || x_stride_head % 8) return HEAL_ERR_INVALID_ARGUMENT;
  if (x_stride_batch < 0 || x_stride_tok < 0 || x_stride_head < 0) return HEAL_ERR_INVALID_ARGUMENT;
  const heal_status_t st = kv_quant_launch(x, x_is_bf16, B, T, H, D, x_stride_batch, x_stride_tok, x_stride_head,
                                           q_cache, scale_cache, Tmax, t_offset, (cudaStream_t)stream);
  if (st == HEAL_ERR_CUDA) (void)cudaGetLastError();
  return st;
}

size_t heal_attention_workspace_bytes_gqa(int B, int Hq, int Hkv, int Tq, int Tmax) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tmax <= 0 || Hq % Hkv != 0) return 0;
  if ((long long)(Hq / Hkv) * Tq <= 8) return attention_workspace_bytes(B, Hq, Tq, Tmax);
  return attention_prefill_workspace_bytes(B, Hq, Hkv, Tq, Tmax);
}

size_t heal_attention_workspace_bytes(int B, int Hq, int Tq, int Tmax) {
  if (B <= 0 || Hq <= 0 || Tq <= 0 || Tmax <= 0) return 0;
  const size_t dec = attention_workspace_bytes(B, Hq, Tq, Tmax);
  if (Tq == 1) return dec;
  // enough for every Hkv that divides Hq (the prefill planes grow with Hkv <= Hq)
  const size_t pre = attention_prefill_workspace_bytes(B, Hq, Hq, Tq, Tmax);
  return pre > dec ? pre : dec;
}

heal_status_t heal_attention_int16(const int16_t* q, const float* q_scale, const int16_t* k_cache,
                                   const float* k_scale, const int16_t* v_cache, const float* v_scale, int B,
                                   int Hq, int Hkv, int D, int Tq, const int32_t* kv_len, int Tmax,
                                   float softmax_scale, int causal, float* out, void* workspace,
                                   size_t workspace_bytes, int64_t* qk_int_out, heal_stream_t stream) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tmax <= 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (Hq % Hkv != 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (D != 64 && D != 128) return HEAL_ERR_UNSUPPORTED;
  const bool prefill = (long long)(Hq / Hkv) * Tq > 8;   // more query rows per KV head than the decode kernel takes
  if (prefill && D != 128) return HEAL_ERR_UNSUPPORTED;
  if (Tmax % 64 != 0) return HEAL_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return HEAL_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale > 0.0f) || softmax_scale != softmax_scale) return HEAL_ERR_INVALID_ARGUMENT;
  if (!q || !q_scale || !k_cache || !k_scale || !v_cache || !v_scale || !kv_len || !out || !workspace)
    return HEAL_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(workspace, 16))
    return HEAL_ERR_INVALID_ARGUMENT;
  if (!aligned(q_scale, 4) || !aligned(k_scale, 16) || !aligned(v_scale, 16) || !aligned(kv_len, 4))
    return HEAL_ERR_INVALID_ARGUMENT;
  if (qk_int_out && !aligned(qk_int_out, 8)) return HEAL_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < heal_attention_workspace_bytes_gqa(B, Hq, Hkv, Tq, Tmax)) return HEAL_ERR_INVALID_ARGUMENT;
  if (prefill) {
    const heal_status_t st =
        attention_prefill_launch(q, q_scale, k_cache, k_scale, v_cache, v_scale, B, Hq, Hkv, Tq, kv_len, Tmax,
                                 softmax_scale, causal, out, workspace, workspace_bytes, qk_int_out, (cudaStream_t)stream);
    if (st == HEAL_ERR_CUDA) (void)cudaGetLastError();
    return st;
  }
  const heal_status_t st = attention_launch(q, q_scale, k_cache, k_scale, v_cache, v_scale, B, Hq, Hkv, D, Tq, kv_len,
                                            Tmax, softmax_scale, causal, out, workspace, workspace_bytes,
                                            qk_int_out, (cudaStream_t)stream);
  if (st == HEAL_ERR_CUDA) (void)cudaGetLastError();
  return st;
}

heal_status_t heal_get_device_status(heal_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return HEAL_ERR_CUDA;
  }
  unsigned int st[2] = {0, 0};
  if (cudaMemcpyFromSymbol(st, g_status, sizeof(st)) != cudaSuccess) {
    (void)cudaGetLastError();
    return HEAL_ERR_CUDA;
  }
  if (st[0] != 0) {
    const unsigned int zero[2] = {0, 0};
    if (cudaMemcpyToSymbol(g_status, zero, sizeof(zero)) != cudaSuccess) {
      (void)cudaGetLastError();
      return HEAL_ERR_CUDA;
    }
    if (st[0] & kStatusTimeout) return HEAL_ERR_TIMEOUT;
    if (st[0] & kStatusBadInput) return HEAL_ERR_INVALID_ARGUMENT;
  }
  return HEAL_OK;
}

heal_status_t heal_probe_wait_timeout(int limit_ms, heal_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 10000) return HEAL_ERR_INVALID_ARGUMENT;
  unsigned int* st = device_status_ptr();
  if (!st) return HEAL_ERR_CUDA;
  heal_wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(st, (unsigned long long)limit_ms * 1000000ull);
  if (cudaGetLastError() != cudaSuccess) return HEAL_ERR_CUDA;
  return HEAL_OK;
}

const char* heal_status_string(heal_status_t s) {
  switch (s) {
    case HEAL_OK: return "ok";
    case HEAL_ERR_INVALID_ARGUMENT: return "invalid argument";
    case HEAL_ERR_UNSUPPORTED: return "unsupported configuration";
    case HEAL_ERR_CUDA: return "CUDA runtime error";
    case HEAL_ERR_TIMEOUT: return "a device-side wait ran out of time";
  }
  return "unknown status";
}

const char* heal_version(void) { return "heal-b200 0.1.0 sm_100a"; }

}  // extern "C"
