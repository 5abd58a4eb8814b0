// Weight-streaming projections of the MFA decode step on the sm_100a tensor cores.
//
// Both hidden-state projections of the layer (Step-3 pages: bud-325 "Method" -- the query
// is down-projected 7168 -> 2048, normalized and up-projected 2048 -> 64 x 256; the shared
// K and V heads are projected 7168 -> 256 each) are skinny GEMMs: a few to a few hundred
// token rows against large weight matrices. Each weight byte is used by every row, so the
// weights are what streams from HBM. They are put on the M side of the MMA ("swap AB"):
//     out^T[n, b] = sum_k W[k, n] * X[b, k]
//   A = W^T tile [128 output features x 128 k] -- read straight from the row-major [in, out]
//       weight by TMA as two [64 features x 128 k] boxes (MN-major, 128-byte swizzle);
//   B = X tile   [N rows x 128 k] as two [N x 64 k] boxes (K-major, 128-byte swizzle), N =
//       batch rounded up to 16;
//   D = TMEM accumulator [128 lanes x N columns] fp32.
// One CTA computes one 128-feature tile over a range of k (split-K for the 7168-long
// reduction of the x-projection), with warp 0 issuing TMA into a multi-stage ring, one
// thread each of warps 1 and 6 issuing the MMAs (even and odd stages, into accumulators of
// their own), and warps 2..5 draining and adding the two accumulators.
// A stage holds 128 k (32 KB of weights, 8 MMAs): each stage costs its MMA thread a barrier
// wait and a commit of several hundred cycles, and at 64 k per stage that overhead, not
// DRAM, set the weight stream's pace. Two issuing threads: one thread keeps about one
// M=128 x N<=32 MMA with fresh shared-memory operands in flight every ~70 cycles, two reach
// the shared-memory operand bandwidth (~40 cycles per MMA); more add nothing. Each ring slot
// belongs to one MMA thread (even slots to the first, odd slots to the second), so every
// slot's barrier phases are waited for by one thread, in order: a parity wait is only
// unambiguous when the waiter is never two phases ahead.
//
// The FP8 path (the step3-fp8 model page: block-fp8 checkpoints; the Step-3 pages: the whole
// model runs in FP8): the weight is stored [out, in] as e4m3 codes with one float32 scale per
// 128 x 128 block, and X arrives as e4m3 codes with one float32 scale per row and 128 k. A
// stage (128 k) is then one [128 features x 128 k] box of weight codes (16 KB) and one
// [N x 128 k] box of X codes, both K-major, and four e4m3 MMAs (K = 32 each) give that
// stage's sum of code products in tensor memory. The two MMA threads again take the ring
// slots of one parity each, and each has up to four buffers of its own, used in turn, so the
// MMAs run ahead of the folding. The block scales differ from stage to stage, so warps 2..5
// fold each stage into registers -- acc[b] += (weight scale * X scale of row b) * D[b] --
// and release the buffer; their sums are the output.
#include <cuda_bf16.h>

#include "mfa_internal.cuh"
#include "sm100.cuh"

namespace mfa {
namespace {

using namespace sm100;

constexpr int kThreads = 224;  // warp 0 TMA, warps 1 and 6 MMA, warps 2..5 epilogue
constexpr int kBK = 128;                // k per stage (two 128-byte swizzle rows of X)
constexpr int kATileBytes = 128 * kBK * 2;  // 32 KB: [128 k rows x 128 B] x 2 boxes
constexpr int kABoxBytes = kATileBytes / 2;
constexpr int kMaxStages = 12;
constexpr size_t kMaxSmem = 232448;  // dynamic shared memory a block may have (227 KB)

constexpr int kMaxW8Kb = 16;    // FP8 path: k blocks per CTA (their scales are staged)
constexpr int kMaxW8Rows = 128;  // FP8 path: X rows per CTA (register accumulators)
constexpr int kMaxDBufs = 8;     // FP8 path: tensor-memory buffers of per-stage sums

struct GemmCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t dfull[kMaxDBufs];  // FP8 path: a stage's sums are in D buffer j
  uint64_t dfree[kMaxDBufs];  // FP8 path: D buffer j read out
  uint64_t acc_full;
  uint32_t tmem_base;
  int32_t abort_flag;
  float wscale[kMaxW8Kb];               // FP8 path: this CTA's weight block scales
  float xscale[kMaxW8Kb][kMaxW8Rows];   // FP8 path: X scales of its rows, per k block
};

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

template <bool kW8>
__global__ void __launch_bounds__(kThreads, 1)
    wgemm_kernel(const __grid_constant__ CUtensorMap w0, const __grid_constant__ CUtensorMap w1,
                 const __grid_constant__ CUtensorMap w2, const __grid_constant__ CUtensorMap xmap,
                 WGemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const int b_box = p.n_box * 128;  // one [N x 64 k] box of bf16 X / [N x 128 k] of e4m3 X
  const int b_bytes = kW8 ? b_box : 2 * b_box;
  constexpr int kSlotBytes = kW8 ? kABoxBytes : kATileBytes;  // weights per stage
  uint8_t* a_ring = base;                                  // stages x kSlotBytes
  uint8_t* b_ring = base + (size_t)stages * kSlotBytes;    // stages x n_box * 256 B
  GemmCtl& C = *reinterpret_cast<GemmCtl*>(b_ring + (size_t)stages * b_bytes);
  volatile int* abort = &C.abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // which weight and which 128 output features
  const int m_abs = p.tile_begin + blockIdx.x;
  const CUtensorMap* wm = &w0;
  int n0 = m_abs * 128;
  int wsel = 0;
  if (p.three_weights) {
    if (m_abs >= p.w0_tiles + p.w1_tiles) {
      wm = &w2;
      n0 = (m_abs - p.w0_tiles - p.w1_tiles) * 128;
      wsel = 2;
    } else if (m_abs >= p.w0_tiles) {
      wm = &w1;
      n0 = (m_abs - p.w0_tiles) * 128;
      wsel = 1;
    }
  }
  const int kb0 = blockIdx.y * p.kblocks_per_cta;
  const int nkb = p.kblocks_per_cta;
  const int b0 = blockIdx.z * (kW8 ? kMaxW8Rows : 256);

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&C.full[i], 1);
      mbar_init(&C.empty[i], 1);
    }
    for (int i = 0; i < kMaxDBufs; ++i) {
      mbar_init(&C.dfull[i], 1);
      mbar_init(&C.dfree[i], 4);  // FP8 path: one arrival per folding warp
    }
    mbar_init(&C.acc_full, 2);  // one commit per MMA thread
    C.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&C.tmem_base, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(wm);
      prefetch_tensormap(&xmap);
      const uint64_t evict_first = policy_evict_first();
      auto load_w = [&](int i) {
        const int s = i % stages, k = (kb0 + i) * kBK;
        uint8_t* a = a_ring + (size_t)s * kSlotBytes;
        if constexpr (kW8) {
          // [128 features x 128 k] codes of the [out, in] weight
          tma_load_2d_hint(a, wm, k, n0, &C.full[s], evict_first);
        } else {
          tma_load_2d_hint(a, wm, n0, k, &C.full[s], evict_first);
          tma_load_2d_hint(a + kABoxBytes, wm, n0 + 64, k, &C.full[s], evict_first);
        }
      };
      constexpr int kWBytes = kW8 ? kABoxBytes : kATileBytes;  // weight bytes per stage
      // The weights depend on no earlier kernel: the first `stages` blocks of them stream in
      // while the previous kernel of the step finishes. X (and the outputs) must wait.
      const int early = stages < nkb ? stages : nkb;
      for (int i = 0; i < early; ++i) {
        mbar_arrive_expect_tx(&C.full[i], kWBytes + b_bytes);
        load_w(i);
      }
      pdl_wait();
      pdl_launch_dependents();
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages, use = i / stages;
        if (i >= early) {
          if (use > 0) mbar_wait(&C.empty[s], (use - 1) & 1, abort);
          if (*abort) break;
          mbar_arrive_expect_tx(&C.full[s], kWBytes + b_bytes);
          load_w(i);
        } else if (*abort) {
          break;
        }
        uint8_t* bs = b_ring + (size_t)s * b_bytes;
        tma_load_2d(bs, &xmap, (kb0 + i) * kBK, b0, &C.full[s]);
        if constexpr (!kW8) tma_load_2d(bs + b_box, &xmap, (kb0 + i) * kBK + 64, b0, &C.full[s]);
        issued = i + 1;
      }
      if (*abort) {
        // stages armed early whose X box was never issued: release the missing bytes, so the
        // phase completes once their weight boxes have landed
        for (int i = issued; i < early; ++i) mbar_complete_tx(&C.full[i], b_bytes);
        const int last = issued > early ? issued : early;
        for (int i = (last > stages ? last - stages : 0); i < last; ++i)
          mbar_wait_drain(&C.full[i % stages], (i / stages) & 1);
      }
    } else {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else if (warp == 1 || warp == 6) {
    pdl_wait();
    pdl_launch_dependents();
    if constexpr (kW8) {
      if (lane == 0) {
        // issuer j: the stages in ring slots of parity j, its k-th into its buffer k mod nbj,
        // once the folding warps have read that buffer's previous stage out
        const int j = warp == 1 ? 0 : 1, nbj = p.dbufs / 2;
        constexpr uint32_t idesc = idesc_f16(128, 0, false, false, false);  // e4m3 x e4m3
        const uint32_t id = idesc | (static_cast<uint32_t>(p.n_box >> 3) << 17);
        int k = 0;
        for (int i = 0; i < nkb; ++i) {
          const int s = i % stages;
          if ((s & 1) != j) continue;
          const int buf = j * nbj + k % nbj;
          mbar_wait(&C.full[s], (i / stages) & 1, abort);
          if (k >= nbj) mbar_wait(&C.dfree[buf], ((k / nbj) - 1) & 1, abort);
          tc_fence_after();
          if (*abort) break;
          const uint32_t a = smem_u32(a_ring + (size_t)s * kSlotBytes);
          const uint32_t b = smem_u32(b_ring + (size_t)s * b_bytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk) {
            const uint64_t ad = sdesc_sw128(a + 32 * kk, 16, 1024);
            const uint64_t bd = sdesc_sw128(b + 32 * kk, 16, 1024);
            umma_f8_ss(tmem + buf * p.n_box, ad, bd, id, kk != 0);
          }
          umma_commit(&C.empty[s]);
          umma_commit(&C.dfull[buf]);
          ++k;
        }
      }
    } else if (lane == 0) {
      // issuer j takes the stages in ring slots of parity j, into accumulator columns
      // [j N, j N + N)
      const int j = warp == 1 ? 0 : 1;
      const uint32_t d = tmem + j * p.n_box;
      // A: W^T straight from the [in, out] weight (MN-major)
      const uint32_t idesc = idesc_f16(128, p.n_box, true, true, false);
      bool first = true;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        if ((s & 1) != j) continue;
        mbar_wait(&C.full[s], (i / stages) & 1, abort);
        tc_fence_after();
        if (*abort) break;
        const uint32_t a = smem_u32(a_ring + (size_t)s * kSlotBytes);
        const uint32_t b = smem_u32(b_ring + (size_t)s * b_bytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(a + 2048 * kk, kABoxBytes, 1024);  // MN-major W^T
          const uint64_t bd = sdesc_sw128(b + (kk >> 2) * b_box + 32 * (kk & 3), 16, 1024);
          umma_f16_ss(d, ad, bd, idesc, !first || kk != 0);
        }
        first = false;
        umma_commit(&C.empty[s]);
      }
      umma_commit(&C.acc_full);
      mbar_wait_drain(&C.acc_full, 0);
    }
  } else {
    pdl_wait();
    pdl_launch_dependents();
    // epilogue: thread = TMEM lane = output feature n0 + row
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    if constexpr (kW8) {
      // the CTA's scales: weight block (n0 / 128, kb0 + i) and X rows b0.. per k block
      // (selected without indexing the parameter arrays, which would copy them to the stack)
      const float* wsc = wsel == 0 ? p.wscale[0] : wsel == 1 ? p.wscale[1] : p.wscale[2];
      const int wld = wsel == 0 ? p.wscale_ld[0] : wsel == 1 ? p.wscale_ld[1] : p.wscale_ld[2];
      const int t = threadIdx.x - 64;  // 0..127
      for (int i = t; i < nkb; i += 128) C.wscale[i] = wsc[(size_t)(n0 / 128) * wld + kb0 + i];
      // the X scales of the CTA's rows: eight independent loads in flight per thread at a time
      // (a load-then-store loop would wait for each load in turn)
      const int n_xs = nkb * p.n_box;
      for (int e0 = 0; e0 < n_xs; e0 += 8 * 128) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * 128 + t, i = e / p.n_box, c = e % p.n_box, b = b0 + c;
          v[u] = (e < n_xs && b < p.batch) ? p.xscale[(size_t)b * p.xscale_ld + kb0 + i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * 128 + t;
          if (e < n_xs) C.xscale[e / p.n_box][e % p.n_box] = v[u];
        }
      }
      named_bar_sync(1, 128);
      float acc[kMaxW8Rows];
#pragma unroll
      for (int c = 0; c < kMaxW8Rows; ++c) acc[c] = 0.f;
      bool ok = true;
      const int nbj = p.dbufs / 2;
      int k0 = 0, k1 = 0;  // stages so far of MMA thread 0 / 1 (ring slots of parity 0 / 1)
      // Stages are folded two at a time, 32 columns per round: the round's four
      // tensor-memory loads are issued before one wait, so their latency is paid once. One
      // lane per warp waits on the barriers (128 threads polling one barrier slow each other
      // down); __syncwarp then orders the rest of the warp after it.
      for (int i = 0; i < nkb; i += 2) {
        const bool two = i + 1 < nkb;
        int buf[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (u == 1 && !two) break;
          const int j = ((i + u) % stages) & 1;
          const int k = j ? k1++ : k0++;
          buf[u] = j * nbj + k % nbj;
          if (lane == 0) mbar_wait(&C.dfull[buf[u]], (k / nbj) & 1, abort);
        }
        __syncwarp();
        if (*abort) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float ws0 = C.wscale[i], ws1 = two ? C.wscale[i + 1] : 0.f;
#pragma unroll
        for (int c0 = 0; c0 < kMaxW8Rows; c0 += 32) {
          if (c0 < p.n_box) {
            const bool hi = c0 + 16 < p.n_box;
            uint32_t r0[16], r1[16], r2[16], r3[16];
            const uint32_t base = tmem + lane_addr + c0;
            tmem_ld_32x32b_x16(base + buf[0] * p.n_box, r0);
            if (hi) tmem_ld_32x32b_x16(base + buf[0] * p.n_box + 16, r1);
            if (two) tmem_ld_32x32b_x16(base + buf[1] * p.n_box, r2);
            if (two && hi) tmem_ld_32x32b_x16(base + buf[1] * p.n_box + 16, r3);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              acc[c0 + j] = fmaf(ws0 * C.xscale[i][c0 + j], __uint_as_float(r0[j]), acc[c0 + j]);
              if (hi)
                acc[c0 + 16 + j] = fmaf(ws0 * C.xscale[i][c0 + 16 + j], __uint_as_float(r1[j]),
                                        acc[c0 + 16 + j]);
              if (two) {
                acc[c0 + j] =
                    fmaf(ws1 * C.xscale[i + 1][c0 + j], __uint_as_float(r2[j]), acc[c0 + j]);
                if (hi)
                  acc[c0 + 16 + j] = fmaf(ws1 * C.xscale[i + 1][c0 + 16 + j],
                                          __uint_as_float(r3[j]), acc[c0 + 16 + j]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&C.dfree[buf[0]]);
          if (two) mbar_arrive(&C.dfree[buf[1]]);
        }
      }
      const int n_abs = m_abs * 128 + row;  // column in the concatenated output
      // by chunks of 16 rows, leaving the loop after the last chunk in use: this code runs
      // once, so every instruction of an unused chunk would be fetched for nothing
#pragma unroll
      for (int c0 = 0; c0 < kMaxW8Rows; c0 += 16) {
        if (!ok || c0 >= p.n_box || b0 + c0 >= p.batch) break;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int b = b0 + c0 + j;
          if (b >= p.batch) break;
          if (p.out_f32 != nullptr)
            p.out_f32[((size_t)blockIdx.y * p.batch + b) * p.out_ld + n_abs] = acc[c0 + j];
          else
            p.out_bf16[(size_t)b * p.out_ld + n_abs] = f32_to_bf16_bits(acc[c0 + j]);
        }
      }
    } else {
    mbar_wait(&C.acc_full, 0, abort);
    tc_fence_after();
    const bool ok = !*abort;
    const int n_abs = m_abs * 128 + row;  // column in the concatenated output
    const bool two = nkb >= 2;  // the second MMA thread's first stage is stage 1
    for (int c0 = 0; c0 < p.n_box; c0 += 16) {
      uint32_t r[16], r1[16];
      tmem_ld_32x32b_x16(tmem + lane_addr + c0, r);
      if (two) tmem_ld_32x32b_x16(tmem + lane_addr + p.n_box + c0, r1);
      tmem_wait_ld();
      if (!ok) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int b = b0 + c0 + i;
        if (b >= p.batch) break;
        const float v = __uint_as_float(r[i]) + (two ? __uint_as_float(r1[i]) : 0.f);
        if (p.out_f32 != nullptr)
          p.out_f32[((size_t)blockIdx.y * p.batch + b) * p.out_ld + n_abs] = v;
        else
          p.out_bf16[(size_t)b * p.out_ld + n_abs] = f32_to_bf16_bits(v);
      }
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && C.abort_flag && p.err != nullptr) atomicOr(p.err, kErrTimeout);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace

int wgemm_n_box(int batch) {
  const int n = batch < 256 ? batch : 256;
  return (n + 15) / 16 * 16;
}

int wgemm_n_box_fp8(int batch) {
  const int n = batch < kMaxW8Rows ? batch : kMaxW8Rows;
  return (n + 15) / 16 * 16;
}

template <bool kW8>
cudaError_t launch_wgemm_t(const CUtensorMap* w, const CUtensorMap& xmap, WGemmArgs p,
                           int m_tiles, int splits, cudaStream_t s) {
  p.n_box = kW8 ? wgemm_n_box_fp8(p.batch) : wgemm_n_box(p.batch);
  const int stage_bytes = (kW8 ? kABoxBytes + p.n_box * 128 : kATileBytes + 2 * p.n_box * 128);
  int stages = static_cast<int>((kMaxSmem - 1024 - sizeof(GemmCtl)) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages > p.kblocks_per_cta) stages = p.kblocks_per_cta;
  if (stages < 2) stages = 2;
  p.stages = stages;
  int cols = 32;
  if (kW8) {
    const int per = 256 / p.n_box < kMaxDBufs / 2 ? 256 / p.n_box : kMaxDBufs / 2;
    p.dbufs = 2 * per;  // per MMA thread: `per` buffers
    while (cols < p.dbufs * p.n_box) cols <<= 1;  // the D buffers
  } else {
    while (cols < 2 * p.n_box) cols <<= 1;  // two accumulators
  }
  p.tmem_cols = cols;
  const size_t smem = 1024 + (size_t)stages * stage_bytes + sizeof(GemmCtl);
  // the limit is set once per device to the most any launch asks for
  static std::atomic<uint64_t> smem_set{0};
  if (smem > (size_t)kMaxSmem ||
      !set_smem_limit_once(reinterpret_cast<const void*>(wgemm_kernel<kW8>), kMaxSmem, &smem_set))
    return cudaErrorInvalidValue;
  const int rows = kW8 ? kMaxW8Rows : 256;
  dim3 grid(m_tiles, splits, (p.batch + rows - 1) / rows);
  return launch_pdl(wgemm_kernel<kW8>, grid, dim3(kThreads), smem, s, w[0], w[1], w[2], xmap,
                    p);
}

cudaError_t launch_wgemm(const CUtensorMap* w, const CUtensorMap& xmap, WGemmArgs p,
                         int m_tiles, int splits, cudaStream_t s) {
  if (p.wscale[0] != nullptr) {
    if (p.kblocks_per_cta > kMaxW8Kb) return cudaErrorInvalidValue;
    return launch_wgemm_t<true>(w, xmap, p, m_tiles, splits, s);
  }
  return launch_wgemm_t<false>(w, xmap, p, m_tiles, splits, s);
}

}  // namespace mfa
