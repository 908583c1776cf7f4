// glue.cu -- K6: the FP32 decoder glue around the compensated GEMMs and the INT16
// attention in a Llama-style block (embedding gather, RMSNorm, rotary position
// embedding, SwiGLU, residual add, greedy argmax).  None of these steps is on the pages;
// they are the plain FP32 operations of the 8B-class decoder the paper evaluates, kept in
// FP32 end to end so that no 16-bit store happens at a kernel boundary (the truncation the
// gist.science technical summary, section 1, identifies as the root cause).
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "heal_internal.h"
#include "heal_ptx.cuh"

// Every kernel here is launched with programmatic dependent launch: it lets the next
// kernel of the stream be scheduled at once and waits for the preceding one before its
// first global access, so only launch and setup overlap the neighbours.

namespace heal {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// out[i, :] = table[ids[i], :]
__global__ void embed_kernel(const float* __restrict__ table, const int32_t* __restrict__ ids, int n, int H,
                             int vocab, float* __restrict__ out, unsigned int* status) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int i = blockIdx.x;
  const int id = ids[i];
  if (id < 0 || id >= vocab) {   // invalid id: zero row and flag it (never read out of bounds)
    if (threadIdx.x == 0 && status) atomicOr(&status[0], kStatusBadInput);
    for (int j = threadIdx.x; j < H; j += blockDim.x) out[(size_t)i * H + j] = 0.0f;
    return;
  }
  const float* src = table + (size_t)id * H;
  for (int j = threadIdx.x; j < H; j += blockDim.x) out[(size_t)i * H + j] = src[j];
}

// y[i, :] = x[i, :] / sqrt(mean(x[i, :]^2) + eps) * w   (sum in a fixed order: per thread,
// then warp shuffles, then warps in index order)
__global__ void rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ w, int H, float eps,
                               float* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  __shared__ float part[kThreads / 32];
  const int i = blockIdx.x;
  const float* xr = x + (size_t)i * H;
  float s = 0.0f;
  for (int j = threadIdx.x; j < H; j += blockDim.x) s = __fmaf_rn(xr[j], xr[j], s);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  float tot = 0.0f;
  for (int k = 0; k < (int)(blockDim.x >> 5); ++k) tot += part[k];
  const float r = rsqrtf(tot / (float)H + eps);
  for (int j = threadIdx.x; j < H; j += blockDim.x) y[(size_t)i * H + j] = xr[j] * r * (w ? w[j] : 1.0f);
}

// Rotary embedding on [n, heads, D] rows (rotate-half convention): for d < D/2,
//   (x[d], x[d + D/2]) <- (x[d] c - x[d + D/2] s, x[d + D/2] c + x[d] s)
// with c = cos_t[pos_i, d], s = sin_t[pos_i, d] from host-made FP32 tables [maxpos, D/2].
__global__ void rope_kernel(float* __restrict__ x, int n, int heads, int D, long long row_stride,
                            const int32_t* __restrict__ pos, const float* __restrict__ cos_t,
                            const float* __restrict__ sin_t) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int i = blockIdx.x / heads, h = blockIdx.x % heads;
  float* r = x + (size_t)i * row_stride + (size_t)h * D;
  const int p = pos[i];
  const int half = D / 2;
  for (int d = threadIdx.x; d < half; d += blockDim.x) {
    const float c = cos_t[(size_t)p * half + d], s = sin_t[(size_t)p * half + d];
    const float a = r[d], b = r[d + half];
    r[d] = a * c - b * s;
    r[d + half] = b * c + a * s;
  }
}

// out[i, j] = silu(g[i, j]) * u[i, j] with g = gu[i, j], u = gu[i, F + j]
__global__ void swiglu_kernel(const float* __restrict__ gu, int n, int F, float* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const long long total = (long long)n * F;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long i = e / F, j = e % F;
    const float g = gu[i * 2 * F + j], u = gu[i * 2 * F + F + j];
    out[e] = (g / (1.0f + expf(-g))) * u;
  }
}

// x += y
__global__ void add_kernel(float* __restrict__ x, const float* __restrict__ y, long long n) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
    x[e] += y[e];
}

// index of the largest value of each row (lowest index among equal maxima; NaN never wins).
// One block of 1024 threads per row: 16-byte loads, four of them in flight per thread
// (a 128256-wide vocabulary row is 31 float4 per thread), then warp shuffles and one pass
// over the 32 warps' candidates.  The order of the comparisons does not matter: the rule
// picks the same index whatever the order.
constexpr int kArgThreads = 1024;
__device__ __forceinline__ void arg_take(float v, int j, float& best, int& idx) {
  if (v > best || (v == best && j < idx)) {
    best = v;
    idx = j;
  }
}
__global__ void __launch_bounds__(kArgThreads) argmax_kernel(const float* __restrict__ x, int rows, int n,
                                                            int32_t* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  __shared__ float wv[kArgThreads / 32];
  __shared__ int wi[kArgThreads / 32];
  const int r = blockIdx.x;
  const float* xr = x + (size_t)r * n;
  float best = -FLT_MAX;
  int idx = 0x7fffffff;
  const bool vec = (n % 4 == 0) && ((reinterpret_cast<uintptr_t>(xr) & 15) == 0);
  if (vec) {
    const float4* x4 = reinterpret_cast<const float4*>(xr);
    const int n4 = n / 4;
    for (int q0 = threadIdx.x; q0 < n4; q0 += 4 * kArgThreads) {
      float4 a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + u * kArgThreads;
        a[u] = q < n4 ? x4[q] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = 4 * (q0 + u * kArgThreads);
        arg_take(a[u].x, j, best, idx);
        arg_take(a[u].y, j + 1, best, idx);
        arg_take(a[u].z, j + 2, best, idx);
        arg_take(a[u].w, j + 3, best, idx);
      }
    }
  } else {
    for (int j0 = threadIdx.x; j0 < n; j0 += 4 * kArgThreads) {
      float a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = j0 + u * kArgThreads < n ? xr[j0 + u * kArgThreads] : -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) arg_take(a[u], j0 + u * kArgThreads, best, idx);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_down_sync(0xffffffffu, best, o);
    const int oi = __shfl_down_sync(0xffffffffu, idx, o);
    arg_take(ov, oi, best, idx);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    wv[w] = best;
    wi[w] = idx;
  }
  __syncthreads();
  if (w == 0) {
    best = wv[lane];
    idx = wi[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_down_sync(0xffffffffu, best, o);
      const int oi = __shfl_down_sync(0xffffffffu, idx, o);
      arg_take(ov, oi, best, idx);
    }
    if (lane == 0) out[r] = idx == 0x7fffffff ? 0 : idx;
  }
}

int grid_for(long long n) {
  const int sms = device_sm_count();
  long long g = (n + kThreads - 1) / kThreads;
  const long long cap = (long long)(sms > 0 ? sms : 148) * 8;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}


// y[b, t, h, :] = x[b, h, t, :]: attention output [B, H, T, D] to token rows [B*T, H*D]
__global__ void heads_to_rows_kernel(const float4* __restrict__ x, float4* __restrict__ y, int H, int T, int D4,
                                     long long rows) {
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const long long r = (long long)blockIdx.x * (blockDim.x / D4) + threadIdx.x / D4;   // source row (b, h, t)
  const int e = threadIdx.x % D4;
  if (r >= rows || threadIdx.x >= (blockDim.x / D4) * D4) return;
  const long long t = r % T, bh = r / T;
  const long long h = bh % H, b = bh / H;
  y[((b * T + t) * H + h) * D4 + e] = x[r * D4 + e];
}

}  // namespace
}  // namespace heal

using namespace heal;

extern "C" {

heal_status_t heal_embedding_gather(const float* table, int vocab, int H, const int32_t* ids, int n, float* out,
                                    heal_stream_t stream) {
  if (n < 0 || H <= 0 || vocab <= 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (n == 0) return HEAL_OK;
  if (!table || !ids || !out) return HEAL_ERR_INVALID_ARGUMENT;
  return launch_pdl(embed_kernel, dim3(n), dim3(kThreads), 0, (cudaStream_t)stream, table, ids, n, H, vocab, out,
                    device_status_ptr()) == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

heal_status_t heal_rmsnorm(const float* x, const float* w, int n, int H, float eps, float* y, heal_stream_t stream) {
  if (n < 0 || H <= 0 || !(eps >= 0.0f)) return HEAL_ERR_INVALID_ARGUMENT;
  if (n == 0) return HEAL_OK;
  if (!x || !y) return HEAL_ERR_INVALID_ARGUMENT;
  return launch_pdl(rmsnorm_kernel, dim3(n), dim3(kThreads), 0, (cudaStream_t)stream, x, w, H, eps, y) == cudaSuccess
             ? HEAL_OK : HEAL_ERR_CUDA;
}

heal_status_t heal_rope(float* x, int n, int heads, int D, int64_t row_stride, const int32_t* pos,
                        const float* cos_t, const float* sin_t, heal_stream_t stream) {
  if (n < 0 || heads <= 0 || D <= 0 || (D & 1) || row_stride < (int64_t)heads * D) return HEAL_ERR_INVALID_ARGUMENT;
  if (n == 0) return HEAL_OK;
  if (!x || !pos || !cos_t || !sin_t) return HEAL_ERR_INVALID_ARGUMENT;
  return launch_pdl(rope_kernel, dim3(n * heads), dim3(64), 0, (cudaStream_t)stream, x, n, heads, D,
                    (long long)row_stride, pos, cos_t, sin_t) == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

heal_status_t heal_swiglu(const float* gate_up, int n, int F, float* out, heal_stream_t stream) {
  if (n < 0 || F <= 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (n == 0) return HEAL_OK;
  if (!gate_up || !out) return HEAL_ERR_INVALID_ARGUMENT;
  return launch_pdl(swiglu_kernel, dim3(grid_for((long long)n * F)), dim3(kThreads), 0, (cudaStream_t)stream, gate_up,
                    n, F, out) == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

heal_status_t heal_add(float* x, const float* y, int64_t n, heal_stream_t stream) {
  if (n < 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (n == 0) return HEAL_OK;
  if (!x || !y) return HEAL_ERR_INVALID_ARGUMENT;
  return launch_pdl(add_kernel, dim3(grid_for(n)), dim3(kThreads), 0, (cudaStream_t)stream, x, y, (long long)n) ==
                 cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

heal_status_t heal_heads_to_rows(const float* x, int B, int H, int T, int D, float* y, heal_stream_t stream) {
  if (B < 0 || H < 0 || T < 0 || D <= 0 || D % 4 != 0 || D > 1024) return HEAL_ERR_INVALID_ARGUMENT;
  const long long rows = (long long)B * H * T;
  if (rows == 0) return HEAL_OK;
  if (!x || !y || x == y) return HEAL_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15u) return HEAL_ERR_INVALID_ARGUMENT;
  const int D4 = D / 4;
  const int per = kThreads / D4 > 0 ? kThreads / D4 : 1;   // source rows per block
  const long long blocks = (rows + per - 1) / per;
  if (blocks >= (1LL << 31)) return HEAL_ERR_UNSUPPORTED;
  return launch_pdl(heads_to_rows_kernel, dim3((unsigned)blocks), dim3(per * D4), 0, (cudaStream_t)stream,
                    reinterpret_cast<const float4*>(x), reinterpret_cast<float4*>(y), H, T, D4, rows) == cudaSuccess
             ? HEAL_OK : HEAL_ERR_CUDA;
}

heal_status_t heal_argmax(const float* x, int rows, int n, int32_t* out, heal_stream_t stream) {
  if (rows < 0 || n <= 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (rows == 0) return HEAL_OK;
  if (!x || !out) return HEAL_ERR_INVALID_ARGUMENT;
  return launch_pdl(argmax_kernel, dim3(rows), dim3(kArgThreads), 0, (cudaStream_t)stream, x, rows, n, out) ==
                 cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

}  // extern "C"
