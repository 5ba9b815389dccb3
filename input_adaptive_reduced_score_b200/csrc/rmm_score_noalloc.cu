// rmm_score_noalloc.cu — rmm_score for callers that cannot allocate device
// memory.
//
// rmm_score needs scratch space for the fp32 partial sums of its row splits,
// which the caller normally allocates and passes in.  Some callers cannot do
// that: an inference-engine plugin that is handed only its input and output
// buffers and must not allocate while it runs, or a serving process whose
// device memory is entirely reserved up front by an external pool, where an
// extra cudaMalloc would fail (and would synchronise the device even when it
// succeeds).  This entry point keeps the scratch in a fixed array that is part
// of the library image instead: every GPU that loads the library holds
// kScratchBytes for it until the process exits.
//
// The caller still passes the activation and the output.  The partial sums
// are overwritten in full by every call before they are read, so nothing in
// the array has to start at zero; all calls share the one array, so calls
// that overlap on the GPU (for example on two streams) race and must be
// serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/rmm.h"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr size_t kScratchBytes = RMM_SCORE_NOALLOC_MAX_BYTES;

// Scratch for the row-split partial sums.  In host code this name is only a
// host-side stand-in for the symbol, never a device address: the kernels get
// the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_score_scratch[kScratchBytes];

// Device address of g_score_scratch on `dev`, looked up once per device with
// that device current; nullptr (and the message set) if the lookup fails.
void* scratch_address(int dev) {
  static std::mutex mu;
  static void* cache[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_score_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("rmm_score_noalloc: cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
      return nullptr;
    }
    cache[dev] = p;
  }
  return cache[dev];
}

}  // namespace
}  // namespace rmm

extern "C" rmm_status rmm_score_noalloc(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                                        int64_t batch_stride, float* ss, int64_t ld_ss, int sqrt_out, void* stream) {
  using namespace rmm;
  clear_error();
  if (dtype != RMM_F32 && dtype != RMM_BF16) {
    set_error("rmm_score_noalloc: dtype %d", dtype);
    return RMM_ERR_UNSUPPORTED;
  }
  if (batch < 1 || batch > 65535 || M < 0 || d < 1 || lda < d || ld_ss < d) {
    set_error("rmm_score_noalloc: bad sizes");
    return RMM_ERR_INVALID_ARG;
  }
  const size_t need = score_workspace_bytes(dtype, batch, M, d);
  if (need > kScratchBytes) {
    set_error("rmm_score_noalloc: this shape needs %zu bytes of partial sums, more than the %zu-byte built-in "
              "scratch; use rmm_score with a caller-provided workspace",
              need, kScratchBytes);
    return RMM_ERR_INVALID_ARG;
  }
  if (M == 0 || need == 0) {
    // no partial sums needed: the plain entry point allocates nothing either
    return rmm_score(A, dtype, batch, M, d, lda, batch_stride, ss, ld_ss, sqrt_out, nullptr, 0, stream);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    set_error("rmm_score_noalloc: no current CUDA device");
    return RMM_ERR_CUDA;
  }
  void* scratch = scratch_address(dev);
  if (!scratch) return RMM_ERR_CUDA;
  return rmm_score(A, dtype, batch, M, d, lda, batch_stride, ss, ld_ss, sqrt_out, scratch, need, stream);
}
