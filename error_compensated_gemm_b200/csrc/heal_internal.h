// heal_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "heal.h"

namespace heal {

// SM count of the current device (cached per device); <= 0 on error.
int device_sm_count();

// Device address of the status word on the current device (nullptr on error).
unsigned int* device_status_ptr();

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, cuuint32_t rank, void* base,
                       const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                       const cuuint32_t* elem_strides, CUtensorMapSwizzle swizzle);

// Launch `kern` with programmatic stream serialization: it may be scheduled before the
// previous kernel on `s` finishes and must call griddepcontrol.wait before reading that
// kernel's results.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Params>(args)...);
}

// The same with a 1-D cluster of `cluster` CTAs (grid.x a multiple of it).
template <typename... Params, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               int cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Params>(args)...);
}

heal_status_t split_launch(const float* x, void* hi, void* lo, long long n, int fmt, cudaStream_t s);

size_t gemm_workspace_bytes(int M, int N, int K, int tile_config);
heal_status_t gemm_launch(int M, int N, int K, const float* A, long long lda, const void* B, long long ldb,
                          float* C, long long ldc, int fmt, const heal_gemm_opts_t& o, cudaStream_t s);

heal_status_t kv_quant_launch(const void* x, int is_bf16, int B, int T, int H, int D, long long sb,
                              long long st, long long sh, int16_t* q, float* sc, int Tmax, int t_off,
                              cudaStream_t s);

size_t attention_workspace_bytes(int B, int Hq, int Tq, int Tmax);
heal_status_t attention_launch(const int16_t* q, const float* qs, const int16_t* k, const float* ks,
                               const int16_t* v, const float* vs, int B, int Hq, int Hkv, int D, int Tq,
                               const int32_t* kv_len, int Tmax, float scale, int causal, float* out,
                               void* ws, size_t ws_bytes, int64_t* qk_out, cudaStream_t s);

// Many query rows per KV head ((Hq/Hkv) * Tq > 8, D = 128): the tcgen05 kernel.
size_t attention_prefill_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tmax);
heal_status_t attention_prefill_launch(const int16_t* q, const float* qs, const int16_t* k, const float* ks,
                                       const int16_t* v, const float* vs, int B, int Hq, int Hkv, int Tq,
                                       const int32_t* kv_len, int Tmax, float scale, int causal, float* out,
                                       void* ws, size_t ws_bytes, int64_t* qk_out, cudaStream_t s);

}  // namespace heal
