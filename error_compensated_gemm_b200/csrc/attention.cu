// attention.cu -- placeholder until the INT16 attention kernel lands.
#include "heal_internal.h"
namespace heal {
size_t attention_workspace_bytes(int B, int Hq, int Tq, int Tmax) { return 16; }
heal_status_t attention_launch(const int16_t*, const float*, const int16_t*, const float*, const int16_t*,
                               const float*, int, int, int, int, int, const int32_t*, int, float, int, float*,
                               void*, size_t, int64_t*, cudaStream_t) {
  return HEAL_ERR_UNSUPPORTED;
}
}  // namespace heal
