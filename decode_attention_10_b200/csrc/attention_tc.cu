// Decode attention of the 64 query heads over the shared K/V head on the sm_100a tensor
// cores (bf16 KV cache).
//
// What it computes (Step-3 pages: bud-325 "Method" -- 64 query heads share ONE K head and
// ONE V head of dimension 256; decode cost is max(attention compute, KV memory access)):
//     out[b][h] = sum_j softmax_j(scale * q[b][h] . K_b[j]) V_b[j],   j < seq_lens[b].
// Because every head reads the same K/V rows, one pass over a sequence's cache serves all
// 64 heads: each cached byte is read from HBM once and used 64 times on chip.
//
// Design (one persistent CTA per SM, warp-specialized):
//   warp 0      TMA producer: Q of the current work item (4 boxes of [64 heads x 64 dims]),
//               then K and V tiles of 128 positions as 16 KB boxes of [128 positions x 64
//               dims] into a 10-slot shared-memory ring (128-byte swizzle).
//   warp 1      TMEM owner and MMA issuer (one thread). Per tile t:
//                 S^T(t)[128 pos x 64 heads] = K(t)[128 x 256] . Q^T        (M=128, N=64)
//                 O^T[256 dims x 64 heads] += V(t)^T[256 x 128] . P^T(t)    (2 x M=128, N=64)
//               S^T is double-buffered in TMEM, so S(t+1) runs while the softmax of t does.
//   warps 2..5  softmax, rescale and epilogue; thread = TMEM lane = one position of the tile
//               (S^T) or one dimension of a half of O^T. Scores live in the log2 domain.
//               The running max m per head is only raised when a tile's max exceeds it by
//               more than 8 (a factor 256); otherwise exponents stay bounded and O needs no
//               rescaling. P^T(t) is written to shared memory as bf16 (MN-major, swizzled).
//   Tiles are windows of 128 positions; the last window of a work item ends at the item's
//   end (it may start before the item or at a negative position, which TMA zero-fills), so
//   rows past a sequence's length are never read. Positions outside the item are masked.
// The split plan (which CTA streams which tiles) is computed on chip: see attn_plan.cuh.
#include <cuda_bf16.h>

#include "attn_plan.cuh"
#include "mfa_internal.cuh"
#include "sm100.cuh"

namespace mfa {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kSlots = 10;             // ring slots (even: a V half-tile's 2 chunks are adjacent)
constexpr int kChunkBytes = 16384;     // [128 positions x 64 dims] bf16
constexpr int kQChunkBytes = 8192;     // [64 heads x 64 dims] bf16
constexpr int kPBytes = 16384;         // P^T: [128 positions x 64 heads] bf16
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemS = 0;         // S^T buffers: columns [0, 64) and [64, 128)
constexpr uint32_t kTmemO = 128;       // O^T halves: columns [128, 192) and [192, 256)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr uint32_t kIdescS = idesc_f16(128, 64, true, false, false);  // K (K-major) x Q (K-major)
constexpr uint32_t kIdescPV = idesc_f16(128, 64, true, true, true);   // V^T (MN) x P^T (MN)

struct __align__(1024) TcSmem {
  uint8_t ring[kSlots][kChunkBytes];
  uint8_t q[4][kQChunkBytes];
  uint8_t p[kPBytes];
  PlanSmem plan;
  float m_used[kHeads];
  float alpha[kHeads];
  float red[4][kHeads];
  float lsum[kHeads];
  uint64_t kv_full[kSlots];
  uint64_t kv_empty[kSlots];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, p_free;
  uint64_t o_free;
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t last_flag;
};

__device__ __forceinline__ int num_tiles(const WorkItem& it) {
  return (it.tok1 - it.tok0 + kTile - 1) / kTile;
}

// Window of tile t of an item: rows [y, y + 128) are loaded, positions [a, e) are used.
__device__ __forceinline__ void tile_window(const WorkItem& it, int t, int& y, int& a, int& e) {
  a = it.tok0 + t * kTile;
  e = min(a + kTile, it.tok1);
  y = (a + kTile <= it.tok1) ? a : it.tok1 - kTile;
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sum 64 per-lane values over the 32 lanes of the warp: afterwards lane l holds the sums of
// entries 2l (in v[0]) and 2l + 1 (in v[1]). Each step exchanges half of the live entries
// with the partner lane (bit 4, 3, 2, 1, 0 of the lane id) and keeps the half it owns.
__device__ __forceinline__ void warp_transpose_sum64(float (&v)[64], int lane) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const bool up = lane & 16;
    const float send = up ? v[i] : v[i + 32];
    const float keep = up ? v[i + 32] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const bool up = lane & 8;
    const float send = up ? v[i] : v[i + 16];
    const float keep = up ? v[i + 16] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = lane & 4;
    const float send = up ? v[i] : v[i + 8];
    const float keep = up ? v[i + 8] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 2;
    const float send = up ? v[i] : v[i + 4];
    const float keep = up ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 1;
    const float send = up ? v[i] : v[i + 2];
    const float keep = up ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
}

// ---------------------------------------------------------------------------------------
// warp 0: TMA producer
// ---------------------------------------------------------------------------------------
__device__ void run_producer(TcSmem& S, const CUtensorMap* q_map, const AttnArgs& a, int g) {
  volatile int* abort = &S.abort_flag;
  uint32_t chunk = 0, issued = 0;
  int item = 0, q_issued = 0;
  prefetch_tensormap(q_map);
  plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem& it) {
    const KvSeq* seq = a.kv + it.b;
    const CUtensorMap* km = &seq->tmap_k;
    const CUtensorMap* vm = &seq->tmap_v;
    if (item > 0) mbar_wait(&S.q_empty, (item - 1) & 1, abort);
    if (!*abort) {
      mbar_arrive_expect_tx(&S.q_full, 4 * kQChunkBytes);
      for (int c = 0; c < 4; ++c) tma_load_2d(S.q[c], q_map, 64 * c, it.b * kHeads, &S.q_full);
      q_issued = item + 1;
    }
    const int n = num_tiles(it);
    auto load_tile = [&](const CUtensorMap* m, int t) {
      int y, a0, e0;
      tile_window(it, t, y, a0, e0);
      for (int c = 0; c < 4; ++c) {
        const uint32_t slot = chunk % kSlots, use = chunk / kSlots;
        if (use > 0) mbar_wait(&S.kv_empty[slot], (use - 1) & 1, abort);
        if (!*abort) {
          mbar_arrive_expect_tx(&S.kv_full[slot], kChunkBytes);
          tma_load_2d(S.ring[slot], m, 64 * c, y, &S.kv_full[slot]);
          issued = chunk + 1;
        }
        ++chunk;
      }
    };
    load_tile(km, 0);
    for (int t = 0; t < n; ++t) {
      if (t + 1 < n) load_tile(km, t + 1);
      load_tile(vm, t);
    }
    ++item;
  });
  // Before the CTA may exit, every copy it started must have landed.
  if (*abort) {
    for (uint32_t c = (issued > kSlots ? issued - kSlots : 0); c < issued; ++c)
      mbar_wait_drain(&S.kv_full[c % kSlots], (c / kSlots) & 1);
    if (q_issued > 0) mbar_wait_drain(&S.q_full, (q_issued - 1) & 1);
  }
}

// ---------------------------------------------------------------------------------------
// warp 1 (one thread): MMA issue
// ---------------------------------------------------------------------------------------
__device__ void run_mma(TcSmem& S, const AttnArgs& a, int g, uint32_t tmem) {
  volatile int* abort = &S.abort_flag;
  uint32_t chunk = 0;
  uint32_t gt = 0;  // tiles issued so far by this CTA (all items)
  int item = 0;
  const uint32_t q_base = smem_u32(S.q[0]);
  plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem& it) {
    const int n = num_tiles(it);
    mbar_wait(&S.q_full, item & 1, abort);
    tc_fence_after();

    auto issue_s = [&](uint32_t tile) {
      const uint32_t j = tile & 1, k = tile >> 1;
      if (k > 0) mbar_wait(&S.s_free[j], (k - 1) & 1, abort);
      tc_fence_after();
      const uint32_t d = tmem + kTmemS + 64 * j;
      for (int c = 0; c < 4; ++c) {
        const uint32_t slot = chunk % kSlots, use = chunk / kSlots;
        mbar_wait(&S.kv_full[slot], use & 1, abort);
        tc_fence_after();
        if (!*abort) {
          const uint32_t a_base = smem_u32(S.ring[slot]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(a_base + 32 * kk, 16, 1024);
            const uint64_t bd = sdesc_sw128(q_base + c * kQChunkBytes + 32 * kk, 16, 1024);
            umma_f16_ss(d, ad, bd, kIdescS, (c | kk) != 0);
          }
          umma_commit(&S.kv_empty[slot]);
        }
        ++chunk;
      }
      if (!*abort) umma_commit(&S.s_full[j]);
    };

    auto issue_pv = [&](uint32_t tile, bool first) {
      mbar_wait(&S.p_full, tile & 1, abort);
      if (first && item > 0) mbar_wait(&S.o_free, (item - 1) & 1, abort);
      tc_fence_after();
      const uint32_t p_base = smem_u32(S.p);
      for (int h = 0; h < 2; ++h) {
        const uint32_t c0 = chunk + 2 * h;
        const uint32_t s0 = c0 % kSlots, s1 = (c0 + 1) % kSlots;
        mbar_wait(&S.kv_full[s0], (c0 / kSlots) & 1, abort);
        mbar_wait(&S.kv_full[s1], ((c0 + 1) / kSlots) & 1, abort);
        tc_fence_after();
        if (!*abort) {
          const uint32_t d = tmem + kTmemO + 64 * h;
          const uint32_t a_base = smem_u32(S.ring[s0]);
#pragma unroll
          for (int kt = 0; kt < kTile / 16; ++kt) {
            const uint64_t ad = sdesc_sw128(a_base + 2048 * kt, kChunkBytes, 1024);
            const uint64_t bd = sdesc_sw128(p_base + 2048 * kt, kPBytes, 1024);
            umma_f16_ss(d, ad, bd, kIdescPV, !(first && kt == 0));
          }
          umma_commit(&S.kv_empty[s0]);
          umma_commit(&S.kv_empty[s1]);
        }
      }
      chunk += 4;
      if (!*abort) umma_commit(&S.p_free);
    };

    for (int t = 0; t < n; ++t) {
      issue_s(gt + t);
      if (t >= 1) issue_pv(gt + t - 1, t - 1 == 0);
    }
    if (!*abort) umma_commit(&S.q_empty);
    issue_pv(gt + n - 1, n == 1);
    gt += n;
    ++item;
  });
  // Every MMA issued must be complete before the tensor memory is released.
  umma_commit(&S.mma_done);
  mbar_wait_drain(&S.mma_done, 0);
}

// ---------------------------------------------------------------------------------------
// split merge (run by the 128 softmax threads of the CTA that finished a sequence last):
//   M[h] = max_i m_i[h],  L[h] = sum_i l_i[h] 2^(m_i[h] - M[h]),
//   out[h][d] = v_mul / L[h] * sum_i 2^(m_i[h] - M[h]) acc_i[h][d].
// The per-split weights are staged in shared memory (the P^T buffer, idle at this point),
// so each thread keeps 2 x 32 independent loads in flight per split.
// ---------------------------------------------------------------------------------------
__device__ void merge_splits(TcSmem& S, const AttnArgs& a, const WorkItem& it, int tid,
                             uint16_t* out, float v_mul) {
  constexpr int kChunkSplits = kPBytes / (sizeof(float) * kHeads);  // 64 splits per pass
  float* w = reinterpret_cast<float*>(S.p);
  const int base = S.plan.slot_base[it.b];
  const int ns = it.nsplit;
  if (tid < kHeads) {
    float M = -INFINITY;
#pragma unroll 4
    for (int i = 0; i < ns; ++i) M = fmaxf(M, __ldcg(partial_m(a.partials, base + i) + tid));
    float L = 0.f;
#pragma unroll 4
    for (int i = 0; i < ns; ++i)
      L += __ldcg(partial_l(a.partials, base + i) + tid) *
           exp2f(__ldcg(partial_m(a.partials, base + i) + tid) - M);
    S.alpha[tid] = M;          // reused as scratch: the merge max
    S.lsum[tid] = v_mul / L;   // and the output scale
  }
  named_bar_sync(1, kSoftmaxThreads);
#pragma unroll 1
  for (int hg = 0; hg < 2; ++hg) {
    float o0[32], o1[32];
#pragma unroll
    for (int h = 0; h < 32; ++h) o0[h] = o1[h] = 0.f;
#pragma unroll 1
    for (int i0 = 0; i0 < ns; i0 += kChunkSplits) {
      const int cnt = min(kChunkSplits, ns - i0);
      for (int e = tid; e < cnt * kHeads; e += kSoftmaxThreads) {
        const int ii = e / kHeads, h = e % kHeads;
        w[e] = exp2f(__ldcg(partial_m(a.partials, base + i0 + ii) + h) - S.alpha[h]);
      }
      named_bar_sync(1, kSoftmaxThreads);
#pragma unroll 1
      for (int ii = 0; ii < cnt; ++ii) {
        const float* src = partial_acc(a.partials, base + i0 + ii) + (hg * 32) * kHeadDim;
        const float* wi = w + ii * kHeads + hg * 32;
        float x0[32], x1[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          x0[h] = __ldcg(src + h * kHeadDim + tid);
          x1[h] = __ldcg(src + h * kHeadDim + 128 + tid);
        }
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          o0[h] = fmaf(wi[h], x0[h], o0[h]);
          o1[h] = fmaf(wi[h], x1[h], o1[h]);
        }
      }
      named_bar_sync(1, kSoftmaxThreads);
    }
#pragma unroll
    for (int h = 0; h < 32; ++h) {
      const int hh = hg * 32 + h;
      out[hh * kHeadDim + tid] = f32_to_bf16_bits(o0[h] * S.lsum[hh]);
      out[hh * kHeadDim + 128 + tid] = f32_to_bf16_bits(o1[h] * S.lsum[hh]);
    }
  }
}

// ---------------------------------------------------------------------------------------
// warps 2..5: softmax, rescale, epilogue, split merge
// ---------------------------------------------------------------------------------------
__device__ void run_softmax(TcSmem& S, const AttnArgs& a, int g, uint32_t tmem) {
  volatile int* abort = &S.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x - 64;        // 0..127
  const int quad = warp & 3;               // TMEM lane quadrant this warp may access
  const int row = quad * 32 + lane;        // tile position / O^T row of this thread
  const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
  const bool fp8 = a.kv_dtype == MFA_KV_FP8_E4M3;
  const float s_mul = a.scale * kLog2e * (fp8 ? a.k_scale : 1.f);
  const float v_mul = fp8 ? a.v_scale : 1.f;
  uint32_t gt = 0;
  int item = 0;
  uint8_t* const p_row = S.p + row * 128;

  plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem& it) {
    const int n = num_tiles(it);
    // this warp's running row sums of heads 2*lane and 2*lane + 1
    float l0 = 0.f, l1 = 0.f;

    for (int t = 0; t < n; ++t) {
      const uint32_t tile = gt + t, j = tile & 1, k = tile >> 1;
      int y, a0, e0;
      tile_window(it, t, y, a0, e0);
      const int pos = y + row;
      const bool valid = pos >= a0 && pos < e0;

      mbar_wait(&S.s_full[j], k & 1, abort);
      tc_fence_after();
      uint32_t sr[kHeads];
      tmem_ld_32x32b_x64(tmem + lane_addr + kTmemS + 64 * j, sr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[j]);

      float s[kHeads];
#pragma unroll
      for (int h = 0; h < kHeads; ++h) s[h] = valid ? __uint_as_float(sr[h]) * s_mul : -INFINITY;

      bool need = (t == 0);
      if (!need) {
#pragma unroll
        for (int h = 0; h < kHeads; ++h) need |= s[h] > S.m_used[h] + kRescaleThreshold;
      }
      if (named_bar_or(1, kSoftmaxThreads, need)) {
        // exact per-head max of this tile across the 128 positions
#pragma unroll
        for (int h = 0; h < kHeads; ++h) {
          const float r = warp_max_f32(s[h]);
          if (lane == 0) S.red[warp - 2][h] = r;
        }
        named_bar_sync(1, kSoftmaxThreads);
        if (tid < kHeads) {
          const float mt = fmaxf(fmaxf(S.red[0][tid], S.red[1][tid]),
                                 fmaxf(S.red[2][tid], S.red[3][tid]));
          const float mo = t == 0 ? -INFINITY : S.m_used[tid];
          const float mn = fmaxf(mo, mt);
          S.alpha[tid] = exp2f(mo - mn);
          S.m_used[tid] = mn;
        }
        named_bar_sync(1, kSoftmaxThreads);
        if (t > 0) {
          l0 *= S.alpha[2 * lane];
          l1 *= S.alpha[2 * lane + 1];
          // O must hold PV(t-1) before it is rescaled
          mbar_wait(&S.p_free, (tile - 1) & 1, abort);
          tc_fence_after();
#pragma unroll 1
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t o[kHeads];
            const uint32_t addr = tmem + lane_addr + kTmemO + 64 * hf;
            tmem_ld_32x32b_x64(addr, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < kHeads; ++h)
              o[h] = __float_as_uint(__uint_as_float(o[h]) * S.alpha[h]);
            tmem_st_32x32b_x64(addr, o);
          }
          tmem_wait_st();
        }
      }

      // probabilities (rounded to bf16, the precision the tensor core reads), the P^T row of
      // this position, and the row sums of the rounded values
      uint32_t pk[kHeads / 2];
#pragma unroll
      for (int h = 0; h < kHeads; h += 2) {
        const float p0 = ex2(s[h] - S.m_used[h]);
        const float p1 = ex2(s[h + 1] - S.m_used[h + 1]);
        const uint32_t w = pack_bf16x2(p0, p1);
        pk[h / 2] = w;
        s[h] = __uint_as_float(w << 16);
        s[h + 1] = __uint_as_float(w & 0xFFFF0000u);
      }
      warp_transpose_sum64(s, lane);
      l0 += s[0];
      l1 += s[1];
      // the P^T buffer is free once PV(t-1) has read it
      if (tile >= 1) mbar_wait(&S.p_free, (tile - 1) & 1, abort);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(p_row + ((c ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full);
    }
    gt += n;

    // ---- epilogue of the item ----
    // row sums: the four warps' partial sums through shared memory
    S.red[warp - 2][2 * lane] = l0;
    S.red[warp - 2][2 * lane + 1] = l1;
    named_bar_sync(1, kSoftmaxThreads);
    if (tid < kHeads) S.lsum[tid] = S.red[0][tid] + S.red[1][tid] + S.red[2][tid] + S.red[3][tid];
    // O^T holds PV of the last tile once its commit has landed
    mbar_wait(&S.p_free, (gt - 1) & 1, abort);
    tc_fence_after();
    // one decision for all 128 threads, so they all take the same barriers below
    const bool ok = !named_bar_or(1, kSoftmaxThreads, *abort != 0);
    uint16_t* out = a.out + (size_t)it.b * kQWidth;
    float* pacc = it.slot >= 0 ? partial_acc(a.partials, it.slot) : nullptr;
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t o[kHeads];
      tmem_ld_32x32b_x64(tmem + lane_addr + kTmemO + 64 * hf, o);
      tmem_wait_ld();
      const int d = hf * 128 + row;
      if (ok) {
        if (it.slot < 0) {
#pragma unroll
          for (int h = 0; h < kHeads; ++h)
            out[h * kHeadDim + d] = f32_to_bf16_bits(__uint_as_float(o[h]) * (v_mul / S.lsum[h]));
        } else {
#pragma unroll
          for (int h = 0; h < kHeads; ++h) pacc[h * kHeadDim + d] = __uint_as_float(o[h]);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.o_free);

    if (it.slot >= 0 && ok) {
      if (tid < kHeads) {
        partial_m(a.partials, it.slot)[tid] = S.m_used[tid];
        partial_l(a.partials, it.slot)[tid] = S.lsum[tid];
      }
      __threadfence();
      named_bar_sync(1, kSoftmaxThreads);
      if (tid == 0) {
        const int old = atomicAdd(a.counters + it.b, 1);
        const int last = old == it.nsplit - 1;
        if (last) atomicExch(a.counters + it.b, 0);
        S.last_flag = last;
      }
      named_bar_sync(1, kSoftmaxThreads);
      if (S.last_flag) {
        __threadfence();
        merge_splits(S, a, it, tid, out, v_mul);
      }
      named_bar_sync(1, kSoftmaxThreads);
    } else {
      named_bar_sync(1, kSoftmaxThreads);
    }
    ++item;
  });
}

__global__ void __launch_bounds__(kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap q_map, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&S.kv_full[i], 1);
      mbar_init(&S.kv_empty[i], 1);
    }
    mbar_init(&S.q_full, 1);
    mbar_init(&S.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], 4);
    }
    mbar_init(&S.p_full, 4);
    mbar_init(&S.p_free, 1);
    mbar_init(&S.o_free, 4);
    mbar_init(&S.mma_done, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  plan_build(S.plan, a.seq_lens, a.kv, a.batch, a.grid, a.err, g == 0);
  for (int b = g; b < a.batch; b += gridDim.x) {
    if (S.plan.len[b] != 0) continue;
    for (int i = threadIdx.x; i < kQWidth; i += kThreads) a.out[(size_t)b * kQWidth + i] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    if (lane == 0) run_producer(S, &q_map, a, g);
  } else if (warp == 1) {
    if (lane == 0) run_mma(S, a, g, tmem);
  } else {
    run_softmax(S, a, g, tmem);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && S.abort_flag) atomicOr(a.err, kErrTimeout);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t attention_tc_smem_bytes() { return sizeof(TcSmem) + 1024; }

cudaError_t launch_attention_tc(const CUtensorMap& q_map, const AttnArgs& a, cudaStream_t s) {
  const size_t smem = attention_tc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attention_tc_kernel<<<a.grid, kThreads, smem, s>>>(q_map, a);
  return cudaGetLastError();
}

}  // namespace mfa
