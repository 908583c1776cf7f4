// attention_noalloc.cu -- heal_attention_int16_noalloc: the INT16 attention call for
// callers that cannot allocate device memory when they call it (serving loops that allow no
// allocation after start-up, plugin hosts that hand over only input and output tensors).
// The scratch that heal_attention_int16 takes from a caller-provided workspace lives here in
// one fixed array of the library's own device memory.
#include <mutex>

#include "heal_internal.h"

namespace heal {
namespace {

// The fixed scratch.  Host code must not use this name as a pointer: on the host it is a
// stand-in, not a device address.  Its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_attn_scratch[HEAL_ATTN_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device, looked up once per device (by the
// first call on that device).  The address is kept for the life of the process: it is not
// looked up again after cudaDeviceReset.
heal_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return HEAL_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return HEAL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return HEAL_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return HEAL_OK;
}

}  // namespace
}  // namespace heal

extern "C" heal_status_t heal_attention_int16_noalloc(const int16_t* q, const float* q_scale,
                                                      const int16_t* k_cache, const float* k_scale,
                                                      const int16_t* v_cache, const float* v_scale, int B, int Hq,
                                                      int Hkv, int D, int Tq, const int32_t* kv_len, int Tmax,
                                                      float softmax_scale, int causal, float* out,
                                                      int64_t* qk_int_out, heal_stream_t stream) {
  // size check first, on the host: the scratch the workspace variant asks for must fit
  if (B <= 0 || Hq <= 0 || Tq <= 0 || Tmax <= 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (Hkv <= 0 || Hq % Hkv != 0) return HEAL_ERR_INVALID_ARGUMENT;
  if (heal_attention_workspace_bytes_gqa(B, Hq, Hkv, Tq, Tmax) > (size_t)HEAL_ATTN_STATIC_SCRATCH_BYTES)
    return HEAL_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const heal_status_t st = heal::scratch_address(&scratch);
  if (st != HEAL_OK) return st;
  return heal_attention_int16(q, q_scale, k_cache, k_scale, v_cache, v_scale, B, Hq, Hkv, D, Tq, kv_len, Tmax,
                              softmax_scale, causal, out, scratch, (size_t)HEAL_ATTN_STATIC_SCRATCH_BYTES,
                              qk_int_out, stream);
}
