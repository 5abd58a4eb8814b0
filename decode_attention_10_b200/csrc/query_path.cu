// Hidden-state projections of the MFA decode step (Step-3 pages: bud-325 "Method" --
// 7168 -> 2048 low-rank query, normalization, 2048 -> 64 x 256; one shared K head and one
// shared V head projected from the same hidden state).
//
//   xproj         partial[s][b][:] = x[b, Ks] [W_qdown | W_k | W_v][Ks, :]   (split-K)
//   xproj_finish  c = sum_s partial;  c_hat = bf16(c * rsqrt(mean(c^2) + eps) * gamma);
//                 k, v = sum_s partial -> bf16 or e4m3(./scale) -> cache row pos[b]
//   q_up          q = bf16(c_hat W_qup)
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

constexpr int kRowsPerBlock = 16;  // token rows per block
constexpr int kKChunk = 64;        // reduction chunk staged in shared memory
constexpr int kColsPerBlock = 128; // one output column per thread

// acc[r] = sum_{k in [k0, k0 + klen)} a[r0 + r][k] * w[k][col] for kRowsPerBlock rows.
__device__ __forceinline__ void rows_dot_column(const uint16_t* __restrict__ a, int lda,
                                                int rows, int r0, const uint16_t* __restrict__ w,
                                                int ldw, int col, int k0, int klen,
                                                float (&acc)[kRowsPerBlock],
                                                float (*a_s)[kKChunk]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = 0.f;
  for (int kc = k0; kc < k0 + klen; kc += kKChunk) {
    __syncthreads();
    for (int i = tid; i < kRowsPerBlock * kKChunk; i += blockDim.x) {
      const int r = i / kKChunk, kk = i % kKChunk;
      const int row = r0 + r;
      a_s[r][kk] = row < rows ? bf16_bits_to_f32(a[(size_t)row * lda + kc + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kKChunk; ++kk) {
      const float wv = bf16_bits_to_f32(w[(size_t)(kc + kk) * ldw + col]);
#pragma unroll
      for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = fmaf(a_s[r][kk], wv, acc[r]);
    }
  }
}

__global__ void __launch_bounds__(kColsPerBlock) xproj_kernel(XProjArgs a) {
  __shared__ float a_s[kRowsPerBlock][kKChunk];
  const int cc = (a.tile_begin + blockIdx.x) * kColsPerBlock + threadIdx.x;  // 0..2559
  const uint16_t* w;
  int ldw, col;
  if (cc < kRank) {
    w = a.w[0], ldw = kRank, col = cc;
  } else if (cc < kRank + kHeadDim) {
    w = a.w[1], ldw = kHeadDim, col = cc - kRank;
  } else {
    w = a.w[2], ldw = kHeadDim, col = cc - kRank - kHeadDim;
  }
  const int split = blockIdx.y;
  const int r0 = blockIdx.z * kRowsPerBlock;
  float acc[kRowsPerBlock];
  rows_dot_column(a.x, kHidden, a.batch, r0, w, ldw, col, split * kXProjKPerSplit,
                  kXProjKPerSplit, acc, a_s);
#pragma unroll
  for (int r = 0; r < kRowsPerBlock; ++r) {
    const int row = r0 + r;
    if (row < a.batch) a.part[((size_t)split * a.batch + row) * kXProjCols + cc] = acc[r];
  }
}

__global__ void __launch_bounds__(kColsPerBlock) q_up_kernel(QUpArgs a) {
  __shared__ float a_s[kRowsPerBlock][kKChunk];
  const int col = blockIdx.x * kColsPerBlock + threadIdx.x;
  const int r0 = blockIdx.z * kRowsPerBlock;
  float acc[kRowsPerBlock];
  rows_dot_column(a.c_hat, kRank, a.batch, r0, a.w_qup, kQWidth, col, 0, kRank, acc, a_s);
#pragma unroll
  for (int r = 0; r < kRowsPerBlock; ++r) {
    const int row = r0 + r;
    if (row < a.batch) a.q[(size_t)row * kQWidth + col] = f32_to_bf16_bits(acc[r]);
  }
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

cudaError_t launch_xproj(const XProjArgs& a, cudaStream_t s) {
  dim3 grid(a.tile_end - a.tile_begin, kXProjSplits, (a.batch + kRowsPerBlock - 1) / kRowsPerBlock);
  xproj_kernel<<<grid, kColsPerBlock, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_xproj_finish(const FinishArgs& a, cudaStream_t s) {
  xproj_finish_kernel<<<a.batch, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_q_up(const QUpArgs& a, cudaStream_t s) {
  dim3 grid(kQWidth / kColsPerBlock, 1, (a.batch + kRowsPerBlock - 1) / kRowsPerBlock);
  q_up_kernel<<<grid, kColsPerBlock, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mfa
