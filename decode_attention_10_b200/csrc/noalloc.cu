// mfa_query_proj_noalloc: the query projection with its scratch memory built into the
// library, for callers that cannot allocate device memory.
//
// Every other compute call takes a workspace that the caller allocates. Some callers have
// no way to do that: a host program whose device memory is planned once at start-up by
// another component (a serving engine that hands all free HBM to its KV cache), code that
// must not call the allocator after start-up because cudaMalloc can synchronize the device
// and take unbounded time, or a plugin interface that passes inputs and outputs but no
// workspace. This entry point needs only the inputs and outputs.
//
// The scratch -- the split-K partials of x W_qdown, the normalized low-rank query and the
// error word -- lives in one file-scope __device__ array of fixed size, sized for at most
// MFA_NOALLOC_MAX_BATCH token rows. The CUDA runtime reserves it on every GPU that loads
// the library, for the life of the process, and zeroes it when it loads the module. Host
// code cannot use the array's name as a device address, so its address is looked up per
// device with cudaGetSymbolAddress (once per device: a device reset, which unloads the
// module, leaves that address stale for the rest of the process).
//
// The partials and c_hat are written before they are read in every call, so only the error
// word must start at zero: it is zero at load, the kernels only OR bits into it, and
// mfa_query_proj_noalloc_get_error reads and clears it.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "mfa_internal.cuh"

namespace mfa {
namespace {

constexpr int kNoAllocMaxBatch = MFA_NOALLOC_MAX_BATCH;
constexpr size_t kNoAllocErr = 0;
constexpr size_t kNoAllocPart = 256;
constexpr size_t kNoAllocPartBytes = sizeof(float) * kXProjSplits * kNoAllocMaxBatch * kXProjCols;
constexpr size_t kNoAllocChat = kNoAllocPart + (kNoAllocPartBytes + 255) / 256 * 256;
constexpr size_t kNoAllocChatBytes = sizeof(uint16_t) * kNoAllocMaxBatch * kRank;
constexpr size_t kNoAllocBytes = kNoAllocChat + (kNoAllocChatBytes + 255) / 256 * 256;

// ~2.3 MiB: x-projection partials [7][32][2560] fp32, c_hat [32][2048] bf16, error word.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
mfa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MFA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MFA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MFA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace mfa

using namespace mfa;

extern "C" MFA_API mfa_status mfa_query_proj_noalloc(const void* x, const void* w_qdown,
                                                     const void* gamma, const void* w_qup,
                                                     float eps, void* q_out, int32_t batch,
                                                     void* stream) {
  if (batch < 1) return MFA_ERR_INVALID_ARG;
  if (batch > kNoAllocMaxBatch) return MFA_ERR_WORKSPACE;
  if (!(eps > 0.f)) return MFA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_qdown, gamma, w_qup, q_out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MFA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  mfa_status st = scratch_address(&scratch);
  if (st != MFA_OK) return st;
  WsLayout L{};
  L.err = kNoAllocErr;
  L.xproj_part = kNoAllocPart;
  L.c_hat = kNoAllocChat;
  L.total = kNoAllocBytes;
  return run_query_proj(x, WRef{w_qdown, nullptr}, gamma, WRef{w_qup, nullptr}, eps, q_out,
                        batch, scratch, L, static_cast<cudaStream_t>(stream));
}

extern "C" MFA_API mfa_status mfa_query_proj_noalloc_get_error(void* stream) {
  void* scratch = nullptr;
  mfa_status st = scratch_address(&scratch);
  if (st != MFA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MFA_ERR_CUDA;
  uint32_t bits = 0;
  uint8_t* word = static_cast<uint8_t*>(scratch) + kNoAllocErr;
  if (cudaMemcpy(&bits, word, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (bits == 0) return MFA_OK;
  if (cudaMemsetAsync(word, 0, sizeof(bits), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MFA_ERR_CUDA;
  return status_of_error_bits(bits);
}

extern "C" MFA_API mfa_status mfa_query_proj_noalloc_wait_selftest(uint32_t limit_us,
                                                                   void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return MFA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  mfa_status st = scratch_address(&scratch);
  if (st != MFA_OK) return st;
  uint32_t* word = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(scratch) + kNoAllocErr);
  return launch_wait_selftest(word, limit_us, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MFA_OK
             : MFA_ERR_CUDA;
}
