// rmm_score_noalloc.cu — rmm_score for callers that cannot allocate device
// memory.
//
// rmm_score needs scratch space for the fp32 partial sums of its row splits
// (fp32 activations, or bf16 whose rows are not 16-byte aligned), which the
// caller normally allocates and passes in.  Some callers cannot do that: an
// inference-engine plugin that is handed only its input and output buffers
// and must not allocate while it runs, or a serving process whose device
// memory is entirely reserved up front by an external pool, where an extra
// cudaMalloc would fail (and would synchronise the device even when it
// succeeds).  This entry point keeps the scratch in a fixed array that is part
// of the library image instead: every GPU that loads the library holds
// kScratchBytes for it until the process exits.  Aligned bf16 input takes the
// one-launch kernel, which needs no scratch at all.
//
// The caller still passes the activation and the output.  The partial sums
// are overwritten in full by every call before they are read, so nothing in
// the array has to start at zero; all calls share the one array, so calls
// that overlap on the GPU (for example on two streams) race and must be
// serialised by the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/rmm.h"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr size_t kScratchBytes = RMM_SCORE_NOALLOC_MAX_BYTES;
constexpr int kMaxDevices = 64;

// Scratch for the row-split partial sums.  In host code this name is only a
// host-side stand-in for the symbol, never a device address: the kernels get
// the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_score_scratch[kScratchBytes];

// Process-unique id of the calling thread's current context (false if none).
// The two driver calls are taken through the runtime's entry-point query, so
// the library keeps no link-time dependency on libcuda.
bool current_context_id(unsigned long long* id) {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  return get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
         get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_score_scratch in the current context of device `dev`.
// The look-up runs once per context: the cache is keyed on the context's
// process-unique id, so after a device reset (a new context, where the array
// may sit elsewhere) the first call looks it up again.  nullptr (and the
// message set) on failure.
void* scratch_address(int dev) {
  static std::mutex mu;
  static struct {
    unsigned long long ctx_id;
    void* ptr;
  } cache[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = 0;
  if (current_context_id(&id) && cache[dev].ptr != nullptr && cache[dev].ctx_id == id) return cache[dev].ptr;
  void* p = nullptr;
  // also binds the device's primary context to this thread if none is current
  const cudaError_t e = cudaGetSymbolAddress(&p, g_score_scratch);
  if (e != cudaSuccess || p == nullptr) {
    set_error("rmm_score_noalloc: cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    return nullptr;
  }
  if (!current_context_id(&id)) {
    set_error("rmm_score_noalloc: no current CUDA context on device %d", dev);
    return nullptr;
  }
  cache[dev].ctx_id = id;
  cache[dev].ptr = p;
  return p;
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
  const size_t need = score_workspace_used(A, dtype, batch, M, d, lda, batch_stride);
  if (need > kScratchBytes) {
    set_error("rmm_score_noalloc: this call needs %zu bytes of partial sums, more than the %zu-byte built-in "
              "scratch; use rmm_score with a caller-provided workspace",
              need, kScratchBytes);
    return RMM_ERR_INVALID_ARG;
  }
  if (need == 0) {
    // no partial sums: rmm_score needs no workspace for this call either
    return rmm_score(A, dtype, batch, M, d, lda, batch_stride, ss, ld_ss, sqrt_out, nullptr, 0, stream);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_error("rmm_score_noalloc: no current CUDA device");
    return RMM_ERR_CUDA;
  }
  void* scratch = scratch_address(dev);
  if (!scratch) return RMM_ERR_CUDA;
  return rmm_score(A, dtype, batch, M, d, lda, batch_stride, ss, ld_ss, sqrt_out, scratch, need, stream);
}
