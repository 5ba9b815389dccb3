// rmm_selftest.cu — checks that the library's bounded waits run out cleanly.
//
// Every wait in librmm's kernels gives up after a fixed time (rmm_device.cuh).
// It then records a site code in the device error word, raises its CTA's
// abort flag so the other roles stop waiting, and lets the kernel return.
// This file makes such waits run out on purpose, on a real GPU, with no
// fault, trap or endless loop involved:
//   0: one thread waits on an mbarrier that nothing arrives on (site 62);
//   1: one thread waits on a global flag that nothing raises (site 63);
//   2: the CTA-pair product whose spare warps would copy B_I.  Its copy
//      counters are preset so that no copy unit is ever handed out.  Every
//      tile's producer then waits for a column block that is never copied.
//      The producer, MMA and epilogue waits give up, and the pair kernel
//      unwinds through its abort path: the drain, the cluster barrier and
//      the release of tensor memory.
// The caller reads the code with rmm_device_error() afterwards; the context
// stays usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/rmm.h"
#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

__global__ void selftest_wait_kernel(int which, const uint32_t* flag, unsigned* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (which == 0)
      mbar_wait(smem_u32(&bar), 0, &abort_flag, err, 62);
    else
      flag_wait_geq(flag, 1u, &abort_flag, err, 63);
  }
  __syncthreads();
}

}  // namespace
}  // namespace rmm

extern "C" rmm_status rmm_selftest_timeout(int which, void* stream) {
  using namespace rmm;
  clear_error();
  if (which < 0 || which > 2) {
    set_error("rmm_selftest_timeout: case %d is not 0, 1 or 2", which);
    return RMM_ERR_INVALID_ARG;
  }
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // one small allocation: the flag / counters, then (case 2) the operands
  constexpr int64_t M = 256, d = 64, N = 256, k = 64;
  constexpr size_t kCtrBytes = 256, kOpBytes = (M * k + d * N + k * N + M * N) * 2 + k * 4;
  void* buf = nullptr;
  cudaError_t e = cudaMallocAsync(&buf, kCtrBytes + kOpBytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(buf, 0, kCtrBytes + kOpBytes, s);
  if (e != cudaSuccess) {
    set_error("rmm_selftest_timeout: allocation: %s", cudaGetErrorString(e));
    return RMM_ERR_CUDA;
  }
  uint32_t* ctr = static_cast<uint32_t*>(buf);
  if (which < 2) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(which, ctr, err);
    e = cudaGetLastError();
  } else {
    // tickets start at 2^31: every copy warp's first ticket is past the last
    // unit (and far from wrapping), so nothing is copied and no block count
    // ever rises
    static const uint32_t kTicket = 0x80000000u;
    e = cudaMemcpyAsync(ctr, &kTicket, sizeof(kTicket), cudaMemcpyHostToDevice, s);
    char* p = static_cast<char*>(buf) + kCtrBytes;
    void* A_I = p;
    void* B = p + M * k * 2;
    void* B_I = p + (M * k + d * N) * 2;
    void* Y = p + (M * k + d * N + k * N) * 2;
    const int32_t* idx = reinterpret_cast<const int32_t*>(p + (M * k + d * N + k * N + M * N) * 2);
    const FusedGather fg{B, N, idx, d, ctr, false, 0};
    if (e == cudaSuccess)
      e = launch_gemm_bf16_tc(A_I, k, B_I, N, M, N, k, Y, RMM_BF16, N, err, s, nullptr, &fg);
  }
  const cudaError_t f = cudaFreeAsync(buf, s);
  if (e == cudaSuccess) e = f;
  if (e != cudaSuccess) {
    set_error("rmm_selftest_timeout: launch: %s", cudaGetErrorString(e));
    return RMM_ERR_CUDA;
  }
  return RMM_OK;
}
