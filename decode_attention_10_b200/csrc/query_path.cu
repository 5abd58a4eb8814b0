// Finish of the hidden-state projection of the MFA decode step (Step-3 pages: bud-325
// "Method" -- the low-rank query is normalized between its down- and up-projection; the
// new token's single K and V vectors are appended to its sequence's cache).
//
// The tensor-core x-projection (gemm_tc.cu) leaves split-K partials of
// x [W_qdown | W_k | W_v]; this kernel, one block per token row:
//   c = sum_s partial[s][b][0:2048];  c_hat = bf16(c * rsqrt(mean(c^2) + eps) * gamma)
//   k, v = sum_s partial[s][b][2048:2560] -> bf16, or e4m3(k / k_scale), e4m3(v / v_scale),
//   written at cache row pos[b] (or seq_lens[b] - 1) of sequence b.
// In a layer step one more block builds the attention's split plan (attn_plan.cuh).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "attn_plan.cuh"
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

constexpr int kFinishThreads = 1024;

// Sum over the block (1024 threads); every thread gets the total.
__device__ __forceinline__ float block_sum_1024(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = red[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

// One block of 1024 threads per token row b. Thread t owns query columns t and t + 1024 and,
// for t < 512, column 2048 + t of [k | v]; all 7 split partials of those columns are loaded
// at once.
__global__ void __launch_bounds__(kFinishThreads) xproj_finish_kernel(FinishArgs a) {
  __shared__ float red[32];
  __shared__ PlanSmem plan;
  // The next kernel (q_up) may launch now: it starts streaming its weights on the SMs the
  // x-projection leaves, and it waits for this grid to complete before it reads c_hat.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (blockIdx.x == a.batch) {
    // The plan block. seq_lens and the KV table were final before the step began, so it
    // does not wait for the x-projection; the attention reads the plan after this grid
    // (and q_up after it) completed.
    plan_build(plan, a.pos, a.kv, a.batch, a.attn_grid, a.err, true);
    plan_store(plan, a.plan, a.batch);
    write_seq_info(plan, a.seq_info, a.batch);
    return;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x, tid = threadIdx.x;
  const float* part = a.part + (size_t)b * kXProjCols;
  const size_t split_stride = (size_t)a.batch * kXProjCols;
  const bool do_q = a.gamma != nullptr;
  const bool do_kv = a.kv != nullptr && tid < 2 * kHeadDim;
  float v0[kXProjSplits], v1[kXProjSplits], vk[kXProjSplits];
#pragma unroll
  for (int sp = 0; sp < kXProjSplits; ++sp) {
    const float* ps = part + sp * split_stride;
    v0[sp] = do_q ? ps[tid] : 0.f;
    v1[sp] = do_q ? ps[tid + kFinishThreads] : 0.f;
    vk[sp] = do_kv ? ps[kRank + tid] : 0.f;
  }
  float c0 = 0.f, c1 = 0.f, ck = 0.f;
#pragma unroll
  for (int sp = 0; sp < kXProjSplits; ++sp) c0 += v0[sp], c1 += v1[sp], ck += vk[sp];
  if (do_q) {
    const float ss = block_sum_1024(fmaf(c0, c0, c1 * c1), red);
    const float r = rsqrtf(ss * (1.0f / kRank) + a.eps);
    uint16_t* ch = a.c_hat + (size_t)b * kRank;
    const uint16_t h0 = f32_to_bf16_bits(c0 * r * bf16_bits_to_f32(a.gamma[tid]));
    const uint16_t h1 =
        f32_to_bf16_bits(c1 * r * bf16_bits_to_f32(a.gamma[tid + kFinishThreads]));
    ch[tid] = h0;
    ch[tid + kFinishThreads] = h1;
    if (a.chat8 != nullptr) {
      // the FP8 path: c_hat (as stored, bf16) quantized per group of 128 columns -- group g
      // is the columns of warps 4 (g mod 8) .. 4 (g mod 8) + 3, in the first half for g < 8
      __shared__ float gmax[32][2];
      const float v0 = bf16_bits_to_f32(h0), v1 = bf16_bits_to_f32(h1);
      float m0 = fabsf(v0), m1 = fabsf(v1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      const int warp = tid >> 5, gw = warp & ~3;
      if ((tid & 31) == 0) {
        gmax[warp][0] = m0;
        gmax[warp][1] = m1;
      }
      __syncthreads();
      const float a0 = fmaxf(fmaxf(gmax[gw][0], gmax[gw + 1][0]), fmaxf(gmax[gw + 2][0], gmax[gw + 3][0]));
      const float a1 = fmaxf(fmaxf(gmax[gw][1], gmax[gw + 1][1]), fmaxf(gmax[gw + 2][1], gmax[gw + 3][1]));
      const float s0 = a0 > 0.f ? __fdiv_rn(a0, 448.f) : 1.f;
      const float s1 = a1 > 0.f ? __fdiv_rn(a1, 448.f) : 1.f;
      uint8_t* q8 = a.chat8 + (size_t)b * kRank;
      q8[tid] = f32_to_e4m3(__fdiv_rn(v0, s0));
      q8[tid + kFinishThreads] = f32_to_e4m3(__fdiv_rn(v1, s1));
      if ((tid & 127) == 0) {
        a.chat8_scale[(size_t)b * (kRank / 128) + (tid >> 7)] = s0;
        a.chat8_scale[(size_t)b * (kRank / 128) + 8 + (tid >> 7)] = s1;
      }
    }
  }
  if (!do_kv) return;
  const int row = a.pos[b] - (a.pos_from_len ? 1 : 0);
  const KvSeq* s = a.kv + b;
  const long long at = kv_row_index(*s, row);  // -1: past the capacity or outside the pool
  if (at < 0) {
    if (tid == 0) atomicOr(a.err, kErrCapacity);
    return;
  }
  const bool is_v = tid >= kHeadDim;
  const int j = is_v ? tid - kHeadDim : tid;
  void* base = is_v ? s->v : s->k;
  if (a.kv_dtype == MFA_KV_BF16) {
    static_cast<uint16_t*>(base)[at * kHeadDim + j] = f32_to_bf16_bits(ck);
  } else {
    const float scale = is_v ? a.v_scale : a.k_scale;
    static_cast<uint8_t*>(base)[at * kHeadDim + j] = f32_to_e4m3(__fdiv_rn(ck, scale));
  }
}

// The FP8 path's activations: one warp per (row, group of 128 values); lane l holds values
// 4 l .. 4 l + 3. scale = max |a| / 448 (1 for an all-zero group), code = e4m3(a / scale),
// both float32 operations rounded to nearest even, the code saturating.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* __restrict__ a,
                                                           int rows, int k,
                                                           uint8_t* __restrict__ codes,
                                                           float* __restrict__ scales) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int groups = k / 128;
  const int task = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (task >= rows * groups) return;
  const int r = task / groups, g = task % groups;
  const size_t off = (size_t)r * k + 128 * g + 4 * lane;
  const uint2 raw = *reinterpret_cast<const uint2*>(a + off);
  const float v[4] = {bf16_bits_to_f32(raw.x & 0xFFFFu), bf16_bits_to_f32(raw.x >> 16),
                      bf16_bits_to_f32(raw.y & 0xFFFFu), bf16_bits_to_f32(raw.y >> 16)};
  float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float sc = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) packed |= static_cast<uint32_t>(f32_to_e4m3(__fdiv_rn(v[i], sc))) << (8 * i);
  *reinterpret_cast<uint32_t*>(codes + off) = packed;
  if (lane == 0) scales[(size_t)r * groups + g] = sc;
}

}  // namespace

cudaError_t launch_quantize_rows(const uint16_t* a, int rows, int k, uint8_t* codes,
                                 float* scales, cudaStream_t s) {
  const int tasks = rows * (k / 128);
  return launch_pdl(quantize_rows_kernel, dim3((tasks + 7) / 8), dim3(256), 0, s, a, rows, k,
                    codes, scales);
}

cudaError_t launch_xproj_finish(const FinishArgs& a, cudaStream_t s) {
  const int blocks = a.batch + (a.plan != nullptr ? 1 : 0);
  return launch_pdl(xproj_finish_kernel, dim3(blocks), dim3(kFinishThreads), 0, s, a);
}

}  // namespace mfa
