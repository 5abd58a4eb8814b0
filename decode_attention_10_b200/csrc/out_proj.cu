// Output projection of the attention side of a decode step: the 64 heads' outputs of one
// token, [64 x 256] = 16384 values, are projected back to the hidden width 7168 (Step-3
// pages: bud-325 "Method" -- the per-token cost counts the linear projections around
// attention, and each layer's attention hands a hidden-width vector to the FFN).
//
// y = bf16(out W_o) runs on the weight GEMM of gemm_tc.cu (W_o^T on the M side, 56 tiles of
// 128 output features, split-K 2 over the 16384-long reduction: 112 CTAs); this file holds
// the split-K finish: y[b][n] = bf16(partial[0][b][n] + partial[1][b][n]).
#include <cuda_bf16.h>

#include "mfa_internal.cuh"

namespace mfa {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

constexpr int kFinishThreads = 256;

// Thread i sums four adjacent columns of both partials; n4 = batch * 7168 / 4.
__global__ void __launch_bounds__(kFinishThreads)
    oproj_finish_kernel(const float* __restrict__ part, uint16_t* __restrict__ y, int n4) {
  // the next kernel may launch now and stream what it does not read from us
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int i = blockIdx.x * kFinishThreads + threadIdx.x;
  if (i >= n4) return;
  const float4 a = __ldcg(reinterpret_cast<const float4*>(part) + i);
  const float4 b = __ldcg(reinterpret_cast<const float4*>(part) + n4 + i);
  uint2 o;
  o.x = pack_bf16x2_rn(a.x + b.x, a.y + b.y);
  o.y = pack_bf16x2_rn(a.z + b.z, a.w + b.w);
  reinterpret_cast<uint2*>(y)[i] = o;
}

}  // namespace

cudaError_t launch_oproj_finish(const float* part, uint16_t* y, int batch, cudaStream_t s) {
  static_assert(kOProjSplits == 2, "the finish sums two partials");
  const int n4 = batch * kHidden / 4;
  const int blocks = (n4 + kFinishThreads - 1) / kFinishThreads;
  return launch_pdl(oproj_finish_kernel, dim3(blocks), dim3(kFinishThreads), 0, s, part, y, n4);
}

}  // namespace mfa
