// Finish of the hidden-state projection of the MFA decode step (Step-3 pages: bud-325
// "Method" -- the low-rank query is normalized between its down- and up-projection; the
// new token's single K and V vectors are appended to its sequence's cache).
//
// The tensor-core x-projection (gemm_tc.cu) leaves split-K partials of
// x [W_qdown | W_k | W_v]; this kernel, one block per token row:
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

// One block per token row: finish the split-K sums, normalize the query half, append K/V.
__global__ void __launch_bounds__(256) xproj_finish_kernel(FinishArgs a) {
  __shared__ float red[8];
  const int b = blockIdx.x, tid = threadIdx.x;
  auto colsum = [&](int c) {
    float s = 0.f;
#pragma unroll
    for (int sp = 0; sp < kXProjSplits; ++sp)
      s += a.part[((size_t)sp * a.batch + b) * kXProjCols + c];
    return s;
  };
  if (a.gamma != nullptr) {
    constexpr int kPer = kRank / 256;
    float c[kPer];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      c[i] = colsum(tid + 256 * i);
      ss = fmaf(c[i], c[i], ss);
    }
    ss = block_sum_256(ss, red);
    const float r = rsqrtf(ss * (1.0f / kRank) + a.eps);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int col = tid + 256 * i;
      a.c_hat[(size_t)b * kRank + col] =
          f32_to_bf16_bits(c[i] * r * bf16_bits_to_f32(a.gamma[col]));
    }
  }
  if (a.kv != nullptr) {
    const float k = colsum(kRank + tid);
    const float v = colsum(kRank + kHeadDim + tid);
    const int row = a.pos[b] - (a.pos_from_len ? 1 : 0);
    const KvSeq* s = a.kv + b;
    const int cap = s->capacity;
    if (row < 0 || row >= cap) {
      if (tid == 0) atomicOr(a.err, kErrCapacity);
      return;
    }
    if (a.kv_dtype == MFA_KV_BF16) {
      static_cast<uint16_t*>(s->k)[(size_t)row * kHeadDim + tid] = f32_to_bf16_bits(k);
      static_cast<uint16_t*>(s->v)[(size_t)row * kHeadDim + tid] = f32_to_bf16_bits(v);
    } else {
      static_cast<uint8_t*>(s->k)[(size_t)row * kHeadDim + tid] = f32_to_e4m3(__fdiv_rn(k, a.k_scale));
      static_cast<uint8_t*>(s->v)[(size_t)row * kHeadDim + tid] = f32_to_e4m3(__fdiv_rn(v, a.v_scale));
    }
  }
}

}  // namespace

cudaError_t launch_xproj_finish(const FinishArgs& a, cudaStream_t s) {
  xproj_finish_kernel<<<a.batch, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mfa
