// mfa_wait_selftest: a check of the failure detection of the decode kernels.
//
// Every wait inside the library's kernels (TMA data landing, MMA completion, the hand-offs
// between warps) is an mbarrier wait bounded by a global-timer limit: when it expires the
// CTA sets an abort flag, stops issuing work, drains what it started and reports
// MFA_ERR_TIMEOUT through the workspace, so that a lost arrival ends the call with an error
// instead of hanging the GPU. This entry point exercises exactly that path on a barrier that
// nothing ever completes, with a short caller-chosen limit, so that a test can check that the
// wait gives up, the error is reported, and the context stays usable.
#include <cuda_runtime.h>

#include "mfa_internal.cuh"
#include "sm100.cuh"

namespace mfa {
namespace {

using namespace sm100;

__global__ void __launch_bounds__(32) wait_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival, which never comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  // every lane waits, as the converged producer and MMA warps do
  const bool done = mbar_wait_limit(&bar, 0, &abort_flag, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0 && (!done || abort_flag)) atomicOr(err, kErrTimeout);
}

}  // namespace
}  // namespace mfa

using namespace mfa;

cudaError_t mfa::launch_wait_selftest(uint32_t* err, uint32_t limit_us, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(err, static_cast<uint64_t>(limit_us) * 1000u);
  return cudaGetLastError();
}

extern "C" MFA_API mfa_status mfa_wait_selftest(void* ws, size_t ws_bytes, uint32_t limit_us,
                                                void* stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < 256)
    return MFA_ERR_INVALID_ARG;
  if (limit_us == 0 || limit_us > 1000000u) return MFA_ERR_INVALID_ARG;
  return launch_wait_selftest(static_cast<uint32_t*>(ws), limit_us,
                              static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MFA_OK
             : MFA_ERR_CUDA;
}
