// Decode attention of the 64 query heads over the shared K/V head -- CUDA-core version.
//
// out[b][h] = sum_j softmax_j(scale * q[b][h] . K_b[j]) V_b[j] (Step-3 pages: bud-325
// "Method"; every query head reads the same single K head and V head, so one pass over a
// sequence's cache serves all 64 heads). Split-K over the cache (flash-decoding): each work
// item of the on-chip plan keeps a running max m and sum l per head (log2 domain) and an
// unnormalized accumulator; items of one sequence are merged by the last CTA to finish.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "attn_plan.cuh"
#include "mfa_internal.cuh"

namespace mfa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 256;
constexpr int kSub = 32;         // positions per shared-memory sub-tile
constexpr int kQPitch = kHeadDim + 1;
constexpr int kKPitch = kHeadDim + 1;
constexpr int kPPitch = kSub + 1;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(hr));
}

struct SimtSmem {
  PlanSmem plan;
  float q[kHeads * kQPitch];
  float k[kSub * kKPitch];
  float v[kSub * kHeadDim];
  float p[kHeads * kPPitch];
  int32_t last;
};

__device__ __forceinline__ float load_kv(const void* base, int dtype, size_t idx) {
  if (dtype == MFA_KV_BF16) return bf16_bits_to_f32(static_cast<const uint16_t*>(base)[idx]);
  return e4m3_to_f32(static_cast<const uint8_t*>(base)[idx]);
}

__global__ void __launch_bounds__(kThreads, 1) attention_simt_kernel(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SimtSmem& S = *reinterpret_cast<SimtSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int g = blockIdx.x;
  plan_build(S.plan, a.seq_lens, a.kv, a.batch, a.grid, a.err, g == 0);

  // zero the output of rejected sequences
  for (int b = g; b < a.batch; b += gridDim.x) {
    if (S.plan.len[b] != 0) continue;
    for (int i = tid; i < kQWidth; i += kThreads) a.out[(size_t)b * kQWidth + i] = 0;
  }

  const bool fp8 = a.kv_dtype == MFA_KV_FP8_E4M3;
  // scores in the log2 domain; the FP8 scales fold into the score scale and the output
  const float s_mul = a.scale * kLog2e * (fp8 ? a.k_scale : 1.f);
  const float v_mul = fp8 ? a.v_scale : 1.f;
  const int h = tid >> 2;    // head owned by this thread
  const int part = tid & 3;  // quarter: positions part*8.. of a sub-tile, dims part + 4 i

  plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem& it) {
    const KvSeq* seq = a.kv + it.b;
    const void* kb = seq->k;
    const void* vb = seq->v;
    __syncthreads();
    for (int i = tid; i < kQWidth; i += kThreads)
      S.q[(i / kHeadDim) * kQPitch + (i % kHeadDim)] =
          bf16_bits_to_f32(a.q[(size_t)it.b * kQWidth + i]);
    float m = -INFINITY, l = 0.f;
    float acc[kHeadDim / 4];
#pragma unroll
    for (int i = 0; i < kHeadDim / 4; ++i) acc[i] = 0.f;

    for (int t0 = it.tok0; t0 < it.tok1; t0 += kSub) {
      const int n = min(kSub, it.tok1 - t0);
      __syncthreads();
      for (int i = tid; i < kSub * kHeadDim; i += kThreads) {
        const int t = i / kHeadDim, d = i % kHeadDim;
        const size_t gi = (size_t)(t0 + t) * kHeadDim + d;
        S.k[t * kKPitch + d] = t < n ? load_kv(kb, a.kv_dtype, gi) : 0.f;
        S.v[t * kHeadDim + d] = t < n ? load_kv(vb, a.kv_dtype, gi) : 0.f;
      }
      __syncthreads();
      float s[8];
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = part * 8 + j;
        float dot = 0.f;
        for (int d = 0; d < kHeadDim; ++d) dot = fmaf(S.q[h * kQPitch + d], S.k[t * kKPitch + d], dot);
        s[j] = t < n ? dot * s_mul : -INFINITY;
        tmax = fmaxf(tmax, s[j]);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      const float m_new = fmaxf(m, tmax);
      const float alpha = exp2f(m - m_new);
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float p = exp2f(s[j] - m_new);
        S.p[h * kPPitch + part * 8 + j] = p;
        psum += p;
      }
      psum += __shfl_xor_sync(0xffffffffu, psum, 1);
      psum += __shfl_xor_sync(0xffffffffu, psum, 2);
      l = l * alpha + psum;
      m = m_new;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kHeadDim / 4; ++i) acc[i] *= alpha;
      for (int t = 0; t < n; ++t) {
        const float p = S.p[h * kPPitch + t];
#pragma unroll
        for (int i = 0; i < kHeadDim / 4; ++i) acc[i] = fmaf(p, S.v[t * kHeadDim + part + 4 * i], acc[i]);
      }
    }

    uint16_t* out = a.out + (size_t)it.b * kQWidth + h * kHeadDim;
    if (it.slot < 0) {
      const float inv = v_mul / l;
#pragma unroll
      for (int i = 0; i < kHeadDim / 4; ++i) out[part + 4 * i] = f32_to_bf16_bits(acc[i] * inv);
      return;
    }
    // partial of a split sequence
    float* pm = partial_m(a.partials, it.slot);
    float* pl = partial_l(a.partials, it.slot);
    float* pa = partial_acc(a.partials, it.slot) + h * kHeadDim;
    if (part == 0) {
      pm[h] = m;
      pl[h] = l;
    }
#pragma unroll
    for (int i = 0; i < kHeadDim / 4; ++i) pa[part + 4 * i] = acc[i];
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int old = atomicAdd(a.counters + it.b, 1);
      const int last = old == it.nsplit - 1;
      if (last) atomicExch(a.counters + it.b, 0);
      S.last = last;
    }
    __syncthreads();
    if (!S.last) return;
    __threadfence();
    // merge the nsplit partials of sequence it.b
    const int base = S.plan.slot_base[it.b];
    float M = -INFINITY;
    for (int i = 0; i < it.nsplit; ++i) M = fmaxf(M, __ldcg(partial_m(a.partials, base + i) + h));
    float L = 0.f;
    for (int i = 0; i < it.nsplit; ++i)
      L += __ldcg(partial_l(a.partials, base + i) + h) *
           exp2f(__ldcg(partial_m(a.partials, base + i) + h) - M);
    float o[kHeadDim / 4];
#pragma unroll
    for (int k = 0; k < kHeadDim / 4; ++k) o[k] = 0.f;
    for (int i = 0; i < it.nsplit; ++i) {
      const float w = exp2f(__ldcg(partial_m(a.partials, base + i) + h) - M);
      const float* src = partial_acc(a.partials, base + i) + h * kHeadDim;
#pragma unroll
      for (int k = 0; k < kHeadDim / 4; ++k) o[k] = fmaf(w, __ldcg(src + part + 4 * k), o[k]);
    }
    const float inv = v_mul / L;
#pragma unroll
    for (int k = 0; k < kHeadDim / 4; ++k) out[part + 4 * k] = f32_to_bf16_bits(o[k] * inv);
  });
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(SimtSmem);
  cudaError_t e = cudaFuncSetAttribute(attention_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attention_simt_kernel<<<a.grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mfa
