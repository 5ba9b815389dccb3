// rmm_attention.cu — reduced attention (work in progress).
#include "rmm_internal.h"

namespace rmm {

size_t attention_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int64_t, int64_t) { return 256; }

cudaError_t launch_attention(const void*, const void*, const void*, int64_t, int64_t, int64_t, int64_t, int64_t,
                             int64_t, int64_t, float, void*, int, int32_t*, int32_t*, float*, float*, void*,
                             unsigned*, cudaStream_t) {
  set_error("reduced attention kernels are not built yet");
  return cudaErrorNotSupported;
}

}  // namespace rmm
