// mfa_split_plan: the length-aware split plan of the decode attention, as the device builds
// it, copied out for inspection. The attention kernels (and the layer step's plan block)
// build the plan in shared memory with plan_build and walk it with plan_get
// (attn_plan.cuh); this kernel runs exactly those functions and writes every CTA's work
// items to a caller buffer, so that the plan's coverage, balance and slot use can be checked
// on what the kernels actually use.
#include <cuda_runtime.h>

#include "attn_plan.cuh"
#include "mfa_internal.cuh"

namespace mfa {
namespace {

constexpr int kItemInts = 8;  // cta, sequence, tok0, tok1, slot, nsplit, split, 0

// One block: build the plan for `grid` CTAs, then list the work items CTA by CTA.
__global__ void __launch_bounds__(1024) split_plan_kernel(const int32_t* seq_lens,
                                                          const KvSeq* kv, int batch, int grid,
                                                          int32_t* out, int max_items) {
  __shared__ PlanSmem P;
  plan_build(P, seq_lens, kv, batch, grid, nullptr, false);
  if (threadIdx.x != 0) return;
  const int NT = P.tile_start[batch];
  int n = 0;
  for (int g = 0; g < grid; ++g) {
    PlanCursor c = plan_begin(P, batch, g);
    WorkItem it;
    while (plan_get(P, batch, c, it)) {
      if (n < max_items) {
        int32_t* o = out + 3 + kItemInts * n;
        o[0] = g, o[1] = it.b, o[2] = it.tok0, o[3] = it.tok1;
        o[4] = it.slot, o[5] = it.nsplit, o[6] = it.split, o[7] = 0;
      }
      ++n;
    }
  }
  out[0] = P.grid;
  out[1] = NT;
  out[2] = n;
}

}  // namespace
}  // namespace mfa

using namespace mfa;

extern "C" MFA_API mfa_status mfa_split_plan(const mfa_kv_cache* kv, const int32_t* seq_lens,
                                             int32_t grid, int32_t* out, size_t out_bytes,
                                             void* stream) {
  if (kv == nullptr || kv->table == nullptr || kv->batch < 1 || kv->batch > kMaxBatch)
    return MFA_ERR_INVALID_ARG;
  if (seq_lens == nullptr || out == nullptr || (reinterpret_cast<uintptr_t>(out) & 3u) != 0)
    return MFA_ERR_INVALID_ARG;
  if (grid < 1 || grid > kMaxAttnGrid) return MFA_ERR_INVALID_ARG;
  const size_t max_items = (size_t)grid + kv->batch;  // each CTA's range ends inside at most
                                                      // one sequence it shares
  if (out_bytes < sizeof(int32_t) * (3 + kItemInts * max_items)) return MFA_ERR_WORKSPACE;
  split_plan_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      seq_lens, static_cast<const KvSeq*>(kv->table), kv->batch, grid, out, (int)max_items);
  return cudaGetLastError() == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}
