// split.cu -- K1: standalone hi/lo split of an FP32 array (used to pre-split constant
// weights once, and to test the split in isolation).  HBM-bound: 4 bytes read and
// 4 bytes written per value.
#include "heal_internal.h"
#include "heal_ptx.cuh"
#include "heal_split.cuh"

namespace heal {

template <int FMT>
__global__ void __launch_bounds__(256) heal_split_kernel(const float* __restrict__ x, uint16_t* __restrict__ hi,
                                                         uint16_t* __restrict__ lo, long long n, int vec,
                                                         unsigned int* status) {
  pdl_launch_dependents();   // programmatic dependent launch: see the launch below
  pdl_wait_prerequisites();  // x may come from the preceding kernel
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  long long tail = 0;
  if (vec) {
    // 8 values per thread per step: two 16-byte loads, one 16-byte store to each output
    const long long n8 = n >> 3;
    for (long long v = gid; v < n8; v += stride) {
      const float4 a = __ldcs(reinterpret_cast<const float4*>(x) + 2 * v);
      const float4 b = __ldcs(reinterpret_cast<const float4*>(x) + 2 * v + 1);
      uint4 h, l;
      h.x = split2<FMT>(a.x, a.y, l.x);
      h.y = split2<FMT>(a.z, a.w, l.y);
      h.z = split2<FMT>(b.x, b.y, l.z);
      h.w = split2<FMT>(b.z, b.w, l.w);
      if (HEAL_DCHECK(8 * v + 8 <= n, status, 410)) {
        __stcs(reinterpret_cast<uint4*>(hi) + v, h);
        __stcs(reinterpret_cast<uint4*>(lo) + v, l);
      }
    }
    tail = n8 << 3;
  }
  for (long long i = tail + gid; i < n; i += stride) {
    uint32_t l;
    const uint32_t h = split2<FMT>(x[i], 0.0f, l);
    if (HEAL_DCHECK(i < n, status, 411)) {
      hi[i] = (uint16_t)(h & 0xFFFFu);
      lo[i] = (uint16_t)(l & 0xFFFFu);
    }
  }
}

heal_status_t split_launch(const float* x, void* hi, void* lo, long long n, int fmt, cudaStream_t s) {
  if (n == 0) return HEAL_OK;
  const int sms = device_sm_count();
  if (sms <= 0) return HEAL_ERR_CUDA;
  const bool vec = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(hi) |
                     reinterpret_cast<uintptr_t>(lo)) & 15) == 0;
  const long long work = vec ? (n >> 3) : n;
  long long blocks = (work + 255) / 256;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  // programmatic dependent launch: scheduled during the preceding kernel, every access
  // after griddepcontrol.wait
  const cudaError_t e =
      fmt == HEAL_SPLIT_FP16_S11
          ? launch_pdl(heal_split_kernel<0>, dim3((unsigned)blocks), dim3(256), 0, s, x, (uint16_t*)hi, (uint16_t*)lo, n,
                       vec ? 1 : 0, device_status_ptr())
          : launch_pdl(heal_split_kernel<1>, dim3((unsigned)blocks), dim3(256), 0, s, x, (uint16_t*)hi, (uint16_t*)lo, n,
                       vec ? 1 : 0, device_status_ptr());
  return e == cudaSuccess ? HEAL_OK : HEAL_ERR_CUDA;
}

}  // namespace heal
