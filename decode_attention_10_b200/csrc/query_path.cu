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
    ch[tid] = f32_to_bf16_bits(c0 * r * bf16_bits_to_f32(a.gamma[tid]));
    ch[tid + kFinishThreads] =
        f32_to_bf16_bits(c1 * r * bf16_bits_to_f32(a.gamma[tid + kFinishThreads]));
  }
  if (!do_kv) return;
  const int row = a.pos[b] - (a.pos_from_len ? 1 : 0);
  const KvSeq* s = a.kv + b;
  if (row < 0 || row >= s->capacity) {
    if (tid == 0) atomicOr(a.err, kErrCapacity);
    return;
  }
  // the row's index in the buffer: the sequence's own rows, or for a paged cache row
  // row % page_size of page pages[row / page_size] of the pool
  size_t at = (size_t)row;
  if (s->page_size != 0) {
    const int page = s->pages[row / s->page_size];
    if (page < 0 || page >= s->num_pages) {
      if (tid == 0) atomicOr(a.err, kErrCapacity);
      return;
    }
    at = (size_t)page * s->page_size + row % s->page_size;
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

}  // namespace

cudaError_t launch_xproj_finish(const FinishArgs& a, cudaStream_t s) {
  const int blocks = a.batch + (a.plan != nullptr ? 1 : 0);
  return launch_pdl(xproj_finish_kernel, dim3(blocks), dim3(kFinishThreads), 0, s, a);
}

}  // namespace mfa
