// Finish of the hidden-state projection of the MFA decode step (Step-3 pages: bud-325
// "Method" -- the low-rank query is normalized between its down- and up-projection; the
// new token's single K and V vectors are appended to its sequence's cache).
//
// The tensor-core x-projection (gemm_tc.cu) leaves split-K partials of
// x [W_qdown | W_k | W_v]; this kernel, nine blocks per token row:
//   c = sum_s partial[s][b][0:2048];  c_hat = bf16(c * rsqrt(mean(c^2) + eps) * gamma)
//   k, v = sum_s partial[s][b][2048:2560] -> bf16, or e4m3(k / k_scale), e4m3(v / v_scale),
//   written at cache row pos[b] (or seq_lens[b] - 1) of sequence b.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "mfa_internal.cuh"

namespace mfa {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ uint8_t f32_to_e4m3(float f) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(f, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < 8 ? red[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);  // all lanes
  return t;
}

// Block (b, j): token row b; j < 8 finishes the query columns [256 j, 256 j + 256) (each of
// these blocks sums the squares of the whole 2048-wide row itself, so no block waits for
// another), j == 8 finishes and appends the K and V rows.
constexpr int kFinishQBlocks = kRank / 256;  // 8

__global__ void __launch_bounds__(256) xproj_finish_kernel(FinishArgs a) {
  __shared__ float red[8];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  const float* part = a.part + (size_t)b * kXProjCols;
  const size_t split_stride = (size_t)a.batch * kXProjCols;
  if (j < kFinishQBlocks) {
    if (a.gamma == nullptr) return;
    constexpr int kPer = kRank / 256;
    float v[kPer][kXProjSplits];
#pragma unroll
    for (int i = 0; i < kPer; ++i)
#pragma unroll
      for (int sp = 0; sp < kXProjSplits; ++sp) v[i][sp] = part[sp * split_stride + tid + 256 * i];
    float ss = 0.f, mine = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      float c = 0.f;
#pragma unroll
      for (int sp = 0; sp < kXProjSplits; ++sp) c += v[i][sp];
      ss = fmaf(c, c, ss);
      if (i == j) mine = c;
    }
    ss = block_sum_256(ss, red);
    const float r = rsqrtf(ss * (1.0f / kRank) + a.eps);
    const int col = tid + 256 * j;
    a.c_hat[(size_t)b * kRank + col] = f32_to_bf16_bits(mine * r * bf16_bits_to_f32(a.gamma[col]));
    return;
  }
  if (a.kv == nullptr) return;
  const int row = a.pos[b] - (a.pos_from_len ? 1 : 0);
  const KvSeq* s = a.kv + b;
  const int cap = s->capacity;
  float kk = 0.f, vv = 0.f;
#pragma unroll
  for (int sp = 0; sp < kXProjSplits; ++sp) {
    kk += part[sp * split_stride + kRank + tid];
    vv += part[sp * split_stride + kRank + kHeadDim + tid];
  }
  if (row < 0 || row >= cap) {
    if (tid == 0) atomicOr(a.err, kErrCapacity);
    return;
  }
  if (a.kv_dtype == MFA_KV_BF16) {
    static_cast<uint16_t*>(s->k)[(size_t)row * kHeadDim + tid] = f32_to_bf16_bits(kk);
    static_cast<uint16_t*>(s->v)[(size_t)row * kHeadDim + tid] = f32_to_bf16_bits(vv);
  } else {
    static_cast<uint8_t*>(s->k)[(size_t)row * kHeadDim + tid] = f32_to_e4m3(__fdiv_rn(kk, a.k_scale));
    static_cast<uint8_t*>(s->v)[(size_t)row * kHeadDim + tid] = f32_to_e4m3(__fdiv_rn(vv, a.v_scale));
  }
}

}  // namespace

cudaError_t launch_xproj_finish(const FinishArgs& a, cudaStream_t s) {
  return launch_pdl(xproj_finish_kernel, dim3(a.batch, kFinishQBlocks + 1), dim3(256), 0, s, a);
}

}  // namespace mfa
