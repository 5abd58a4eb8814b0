// Decode attention of the 64 query heads over the shared K/V head on the sm_100a tensor
// cores, for bf16 and FP8 (e4m3) KV caches.
//
// What it computes (Step-3 pages: bud-325 "Method" -- 64 query heads share ONE K head and
// ONE V head of dimension 256; decode cost is max(attention compute, KV memory access)):
//     out[b][h] = sum_j softmax_j(scale * q[b][h] . K_b[j]) V_b[j],   j < seq_lens[b].
// Because every head reads the same K/V rows, one pass over a sequence's cache serves all
// 64 heads: each cached byte is read from HBM once and used 64 times on chip.
//
// Design (one persistent CTA per SM, warp-specialized, 320 threads; 352 for FP8 caches):
//   warp 0      TMA producer: Q of each work item (4 boxes of [64 heads x 64 dims]; two Q
//               buffers, so the next item's Q loads while this one streams), then K and V
//               tiles of 128 positions as 16 KB boxes of [128 positions x 64 dims] into a
//               6-slot shared-memory ring (128-byte swizzle).
//   warp 1      TMEM owner and MMA issuer (one elected lane; the warp runs converged). Per
//               tile t:
//                 S^T(t)[128 pos x 64 heads] = K(t)[128 x 256] . Q^T        (M=128, N=64)
//                 O^T[256 dims x 64 heads] += V(t)^T[256 x 128] . P^T(t)    (2 x M=128, N=64)
//               S^T is double-buffered in TMEM, so S(t+1) runs while the softmax of t does.
//   warps 2..9  softmax, rescale and epilogue, in two groups of four warps: group 0 owns
//               heads 0..31, group 1 heads 32..63, of the same tile. Thread = TMEM lane =
//               one position of the tile (S^T) or one dimension of a half of O^T. Scores
//               live in the log2 domain. The running max m per head is only raised when a
//               tile's max exceeds it by more than 8 (a factor 256); otherwise exponents stay
//               bounded and O needs no rescaling. Each group writes its heads' half of the
//               P^T(t) row (16-bit, MN-major, swizzled). The groups share no state, so
//               neither waits for the other except through the MMA barriers.
//   Tiles are windows of 128 positions; the last window of a work item ends at the item's
//   end (it may start before the item or at a negative position, which TMA zero-fills), so
//   rows past a sequence's length are never read. Positions outside the item are masked.
// FP8 caches: the e4m3 codes go to the tensor cores as they are (tcgen05 kind::f8f6f4; e4m3
// values times the power-of-two scales below are exact, and so are the products). The ring
// holds raw boxes of [128 positions x 128 dims] (128 bytes a row, the same swizzle), two per
// K or V tile: a 4-box K ring read by warp 1, which issues the S products, and a 4-box V ring
// read by warp 10, which issues the PV products (an issuing thread waits while the tensor
// core's queue is full, so with one issuing warp a PV whose P was ready waited behind the
// issue of the next S). Each S and each PV is issued as 8 MMAs back to back once both of its
// boxes have landed. The other operand must be e4m3 too, so Q and P each become a
// pair of e4m3 matrices with one common scale, a high part and the rounded remainder (hi +
// lo keeps 7 to 8 significant bits, about what bf16 keeps), stacked along N:
//   S^T(t)[128 pos x 128] = K(t) . [Q_hi ; Q_lo]^T        (M=128, N=128: hi heads, lo heads)
//   O^T[256 x 128]     += V(t)^T . [P_hi | P_lo]^T(t)  (2 x M=128, N=128)
// and the softmax adds the two halves of S, the epilogue those of O. Q is split once per
// work item by the softmax warps (scaled by 2^-e so that its largest magnitude is in
// [128, 256)), the next item's at the end of the current one; P is computed as
// 2^(s - m + 4) and raised m only when a tile's max exceeds it by more than 4, so P stays
// below 2^8 and its useful values clear e4m3's subnormal range. The K and V scales fold into
// the softmax scale and the output scale.
// The split plan (which CTA streams which tiles) is computed on chip: see attn_plan.cuh.
// A sequence covered by one CTA is finished in place; the items of a sequence split over
// several CTAs leave (m, l, acc) partials that attention_combine_kernel merges.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_plan.cuh"
#include "mfa_internal.cuh"
#include "sm100.cuh"

namespace mfa {
namespace {

using namespace sm100;

constexpr int kGroupThreads = 128;      // one softmax group = four warps = the 128 lanes
constexpr int kMaxSoftmaxWarps = 16;
// a ring box: [128 positions x 128 bytes] (64 bf16 dims, or 128 e4m3 dims), 128-byte swizzle
constexpr int kChunkBytes = 16384;
constexpr int kRingBytes = 10 * kChunkBytes;
constexpr int kMaxSlots = 10;
constexpr int kQChunkBytes = 8192;      // bf16 Q box: [64 heads x 64 dims]
constexpr int kQ8ChunkBytes = 16384;    // FP8 Q: [128 rows (hi, then lo) x 128 dims] e4m3
constexpr int kPBytes = 16384;          // P^T: [128 positions x 128 bytes]
constexpr uint32_t kTmemS = 0;          // S^T buffers from column 0 (see Cfg::kSCols)
constexpr int kPageIds = 128;          // paged caches: page ids held per work item
constexpr float kLog2e = 1.4426950408889634f;
// named barriers: 1 + group among one softmax group, Cfg::kBarAll among all softmax warps

// Per cache type. bf16 caches: a 6-slot ring of [128 positions x 64 dims] boxes (four per K
// or V tile); S^T and each O^T half are 64 columns (N = 64 heads). FP8 caches: an 8-slot
// ring of [128 positions x 128 dims] e4m3 boxes (two per K or V tile); S^T and each O^T half
// are 128 columns (the hi parts of the 64 heads, then the lo parts), and P =
// 2^(s - m + kPExp). Both: a second Q buffer in the rest of the ring area, and two softmax
// groups of 32 heads (four groups of 16 heads were measured slower for FP8: the extra warps
// slowed the MMA warp's issue more than they sped up the softmax). A softmax group is four
// warps, one per tensor-memory lane quadrant, so that together they hold the 128 positions
// of a tile.
template <bool kFp8>
struct Cfg {
  static constexpr int kGroups = 2;
  static constexpr int kSoftmaxWarps = 4 * kGroups;     // warps 2 .. 2 + kSoftmaxWarps - 1
  // FP8: S and PV are issued by two warps (warp 1 and warp kPvWarp), so that a PV is never
  // held back behind the issue of the next S (an issuing thread waits while the tensor core's
  // queue is full); K and V boxes then sit in rings of their own, each read by one warp
  static constexpr bool kSplitIssue = kFp8;
  static constexpr int kPvWarp = 2 + kSoftmaxWarps;
  static constexpr int kMmaWarps = kSplitIssue ? 2 : 1;
  static constexpr int kThreads = 64 + 32 * kSoftmaxWarps + (kSplitIssue ? 32 : 0);
  // the launch bound: at most three warps share an SM sub-partition, so 168 registers a thread
  // is the ceiling either way (384 threads cap the compiler at it)
  static constexpr int kBoundThreads = kSplitIssue ? 384 : kThreads;
  static constexpr int kGroupHeads = kHeads / kGroups;  // heads per group
  static constexpr uint32_t kBarAll = 1 + kGroups;      // named barrier of all softmax warps
  // bf16 ring: even, so a V half-tile's 2 chunks are adjacent. FP8: K boxes in slots
  // [0, kKSlots), V boxes in [kKSlots, kSlots)
  static constexpr int kSlots = kFp8 ? 8 : 6;
  static constexpr int kKSlots = kSplitIssue ? 4 : kSlots;
  static constexpr int kTileBoxes = kFp8 ? 2 : 4;   // ring boxes per K (or V) tile
  static constexpr int kBoxDims = kFp8 ? 128 : 64;  // head dims per box
  static constexpr int kMmaK = kFp8 ? 32 : 16;      // K of one MMA instruction
  static constexpr uint32_t kTmemCols = kFp8 ? 512 : 256;
  static constexpr uint32_t kSCols = kFp8 ? 128 : 64;  // S^T buffer, or O^T half, columns
  static constexpr uint32_t kTmemO = 2 * kSCols;       // O^T halves follow the S^T buffers
  static constexpr int kQBufs = 2;
  static constexpr int kQ1Off = kSlots * kChunkBytes;  // the second Q buffer in the ring area
  static constexpr float kRescaleThreshold = kFp8 ? 4.0f : 8.0f;  // log2 units
  static constexpr float kPExp = kFp8 ? 4.0f : 0.0f;  // P = 2^(s - m + kPExp)
  // operand formats: bf16 (kind::f16), or e4m3 (kind::f8f6f4, whose format code is 0)
  static constexpr uint32_t kIdescS = idesc_f16(128, kSCols, !kFp8, false, false);  // K x Q^T
  static constexpr uint32_t kIdescPV = idesc_f16(128, kSCols, !kFp8, true, true);   // V^T x P^T
};
static_assert(Cfg<true>::kSlots <= kMaxSlots && Cfg<false>::kSlots <= kMaxSlots, "ring");
static_assert(!Cfg<true>::kSplitIssue ||
                  (Cfg<true>::kPvWarp * 32 + 32 == Cfg<true>::kThreads &&
                   Cfg<true>::kThreads <= Cfg<true>::kBoundThreads && Cfg<true>::kKSlots % 2 == 0),
              "FP8: the PV warp is the last warp; K and V rings of whole tiles");
static_assert(Cfg<false>::kPvWarp * 32 == Cfg<false>::kThreads, "bf16: no PV warp");
static_assert(2 * kQ8ChunkBytes == 4 * kQChunkBytes, "FP8 Q is split in place");
static_assert(Cfg<true>::kSoftmaxWarps <= kMaxSoftmaxWarps &&
                  Cfg<false>::kSoftmaxWarps <= kMaxSoftmaxWarps,
              "softmax warps");
static_assert(Cfg<true>::kBarAll < 16 && Cfg<false>::kBarAll < 16, "named barrier ids");
static_assert(Cfg<false>::kQ1Off + 4 * kQChunkBytes <= kRingBytes, "second Q buffer (bf16)");
static_assert(Cfg<true>::kQ1Off + 4 * kQChunkBytes <= kRingBytes, "second Q buffer (FP8)");

struct __align__(1024) TcSmem {
  uint8_t ring_area[kRingBytes];
  uint8_t q[4][kQChunkBytes];
  uint8_t p[kPBytes];
  PlanSmem plan;
  float m_used[kHeads];
  float m_thr[kHeads];  // m_used + the rescale threshold: a score above it needs a rescale
  float m_p[kHeads];    // m_used - the P exponent offset: P = 2^(s - m_p)
  float alpha[kHeads];
  float red[4][kHeads];
  float lsum[kHeads];
  float qmax[kMaxSoftmaxWarps];
  uint64_t kv_full[kMaxSlots];
  uint64_t kv_empty[kMaxSlots];
  uint64_t q_full[2], q_empty[2];
  uint64_t q_ready;  // FP8: Q split into its e4m3 hi and lo parts
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, p_free;
  uint64_t o_free;
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t page_ids[2][kPageIds];  // paged caches: the first page ids of this and the next item
};

// the dynamic shared memory of one CTA (TcSmem plus its 1024-byte alignment) fits the
// 227 KB a block may have
static_assert(sizeof(TcSmem) + 1024 <= 232448, "shared memory per CTA");

// ring box `slot`
__device__ __forceinline__ uint8_t* ring_chunk(TcSmem& S, uint32_t slot) {
  return S.ring_area + slot * kChunkBytes;
}
// Q buffer qb: [4 boxes of 64 heads x 64 dims] bf16 as loaded (for FP8 caches then split in
// place into 2 chunks of [128 rows x 128 dims] e4m3)
template <bool kFp8>
__device__ __forceinline__ uint8_t* q_buf(TcSmem& S, int qb) {
  return qb == 0 ? S.q[0] : S.ring_area + Cfg<kFp8>::kQ1Off;
}

__device__ __forceinline__ int num_tiles(const WorkItem& it) {
  return (it.tok1 - it.tok0 + kTile - 1) / kTile;
}

// Window of tile t of an item: rows [y, y + 128) are loaded, positions [a, e) are used.
// Contiguous caches: an item's last window slides back to end at the item's end, so no row
// past the sequence is read (rows before a are the sequence's own, or zero-filled below row
// 0). Paged caches: windows stay on 128-position boundaries, so each 64-row half lies in one
// page; rows [e, y + 128) past the sequence's end are loaded (from its last page, or zeros
// past it) and their V values zeroed on chip.
__device__ __forceinline__ void tile_window(const WorkItem& it, int t, bool paged, int& y,
                                            int& a, int& e) {
  a = it.tok0 + t * kTile;
  e = min(a + kTile, it.tok1);
  y = (paged || a + kTile <= it.tok1) ? a : it.tok1 - kTile;
}

// Paged caches: rows of a window whose V values are used (the rest are zeroed before PV).
__device__ __forceinline__ int window_rows_kept(bool paged, int y, int e) {
  return paged ? e - y : kTile;
}

// Zero rows [from, 128) of a [128 x 128 B] 16-bit chunk (row r is bytes [128 r, 128 r + 128)
// whatever the swizzle), by the 32 lanes of a warp.
__device__ __forceinline__ void zero_chunk_rows(uint8_t* chunk, int from, int lane) {
  uint4* p = reinterpret_cast<uint4*>(chunk + from * 128);
  const int n = (kTile - from) * 8;
  for (int i = lane; i < n; i += 32) p[i] = make_uint4(0u, 0u, 0u, 0u);
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

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sum N (32 or 16) per-lane values over the 32 lanes of the warp. Each step exchanges half
// of the live entries with the partner lane (bit 4, 3, ... of the lane id) and keeps the
// half it owns; once one entry is left, the remaining steps are plain sums. Afterwards lane
// l holds the sum of entry l (N = 32) or of entry l / 2 (N = 16, lanes l and l ^ 1 alike).
template <int N>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[N], int lane) {
  static_assert(N == 32 || N == 16, "entries");
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int bit = 16 >> step;
    const int live = N >> step;  // entries still live before this step (>= 1)
    if (live >= 2) {
      const int half = live / 2;
      const bool up = lane & bit;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], bit);
    }
  }
  return v[0];
}

// tensor memory: N = 32 or 16 consecutive columns of this warp's 32 lanes
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 32)
    tmem_ld_32x32b_x32(taddr, r);
  else
    tmem_ld_32x32b_x16(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 32)
    tmem_st_32x32b_x32(taddr, r);
  else
    tmem_st_32x32b_x16(taddr, r);
}

// ---------------------------------------------------------------------------------------
// warp 0: TMA producer
// ---------------------------------------------------------------------------------------
template <bool kFp8, bool kPaged>
__device__ void run_producer(TcSmem& S, const CUtensorMap* q_map, const AttnArgs& a, int g,
                             bool leader) {
  using C = Cfg<kFp8>;
  constexpr uint32_t kN = C::kSlots;
  volatile int* abort = &S.abort_flag;
  const int lane = threadIdx.x & 31;
  constexpr bool paged = kPaged;
  const int page_size = kPaged ? S.plan.page_size : 1;  // read only by the paged code
  const int page_shift = 31 - __clz(page_size);         // page sizes are powers of two
  const int box_rows = kPaged ? paged_box_rows(page_size) : kTile;
  constexpr int kC = C::kTileBoxes;
  uint32_t chunk = 0, issued = 0;  // ring boxes (FP8: the K ring's)
  uint32_t vchunk = 0, vissued = 0;  // FP8: the V ring's
  constexpr uint32_t kKN = C::kKSlots;
  constexpr uint32_t kVN = kN > C::kKSlots ? kN - C::kKSlots : 1;  // (unused with one ring)
  int item = 0, q_issued = 0;
  if (leader) prefetch_tensormap(q_map);
  // every K/V byte is read once: keep it from evicting q and the split partials from L2
  const uint64_t evict_first = policy_evict_first();

  // the current work item and the next one, whose tensor maps are fetched while the
  // current one streams
  PlanCursor cur = plan_begin(S.plan, a.batch, g);
  WorkItem it, nx;
  bool has = plan_get(S.plan, a.batch, cur, it);
  bool has_nx = has && plan_get(S.plan, a.batch, cur, nx);
  if (has && leader) {
    prefetch_tensormap(&a.kv[it.b].tmap_k);
    prefetch_tensormap(&a.kv[it.b].tmap_v);
  }
  // The boxes of one item in the order the MMA consumes them -- K(0), then K(t+1), V(t) for
  // each t, then V(n-1) -- as kC boxes of [128 positions x 128 bytes] per K or V tile,
  // straight into the ring.
  constexpr int kBoxesPerTile = 2 * kC;
  // Paged caches: the page ids of work item k, pages [p0, p_last] of its sequence (p_last =
  // the page of its last position), sit in S.page_ids[k & 1] (the first kPageIds of them; the
  // leader reads any further id straight from the table). Each lane fetches its share of the
  // next item's ids into registers while the current item streams, and stores them when
  // that item begins, so no copy waits for the page table.
  constexpr int kIdsPerLane = kPageIds / 32;
  int32_t ids_next[kIdsPerLane];
  auto first_page = [&](const WorkItem& w) { return w.tok0 >> page_shift; };
  auto last_page = [&](const WorkItem& w) { return (w.tok1 - 1) >> page_shift; };
  auto fetch_ids = [&](const WorkItem& w) {
    const int32_t* pages = a.kv[w.b].pages;
    const int p0 = first_page(w), n = last_page(w) - p0 + 1;
#pragma unroll
    for (int k = 0; k < kIdsPerLane; ++k) {
      const int i = lane + 32 * k;
      ids_next[k] = i < n ? pages[p0 + i] : 0;
    }
  };
  auto store_ids = [&](int buf) {
    __syncwarp();
#pragma unroll
    for (int k = 0; k < kIdsPerLane; ++k) S.page_ids[buf][lane + 32 * k] = ids_next[k];
    __syncwarp();
  };
  // one box of 128 rows at window row y: a 2-D load, or for a paged cache 128 / box_rows
  // 3-D loads of box_rows rows, each from its page. Every lane makes the page lookups (the
  // refills are warp-wide); the leader issues the copies if ok.
  auto load_rows = [&](uint8_t* dst, const CUtensorMap* map, int x, const WorkItem& w, int y,
                       uint64_t* bar, uint64_t policy, bool ok) {
    if constexpr (!kPaged) {
      if (leader && ok) tma_load_2d_hint(dst, map, x, y, bar, policy);
    } else {
      // rows past the item's last page (the sequence's end) are read from that page at a
      // row >= page_size, which the tensor map fills with zeros
      const int p0 = first_page(w), pl = last_page(w);
      for (int r0 = 0; r0 < kTile; r0 += box_rows) {
        const int pos = y + r0;  // >= 0: paged windows start on tile boundaries
        const int pidx = min(pos >> page_shift, pl);
        if (leader && ok) {
          const int i = pidx - p0;
          const int page = i < kPageIds ? S.page_ids[item & 1][i] : a.kv[w.b].pages[pidx];
          tma_load_3d_hint(dst + r0 * 128, map, x, pos - (pidx << page_shift), page, bar, policy);
        }
      }
    }
  };
  // box j of an item: K or V, of tile t, column box c
  auto classify = [&](const WorkItem& w, int j, bool& is_v, int& t, int& c) {
    const int n = num_tiles(w);
    if (j < kC) {
      is_v = false, t = 0, c = j;
    } else {
      const int rr0 = j - kC, tt = rr0 / (2 * kC), rr = rr0 % (2 * kC);
      if (tt < n - 1)
        is_v = rr >= kC, t = is_v ? tt : tt + 1, c = is_v ? rr - kC : rr;
      else
        is_v = true, t = n - 1, c = rr;
    }
  };
  auto issue_box = [&](const WorkItem& w, int j) {
    const KvSeq* seq = a.kv + w.b;
    int y, a0, e0;
    bool is_v;
    int t, c;
    classify(w, j, is_v, t, c);
    tile_window(w, t, paged, y, a0, e0);
    // the box's slot and the use of that slot it is (one ring, or FP8's K and V rings)
    uint32_t slot, use;
    uint32_t* rc = &chunk;
    if constexpr (C::kSplitIssue) {
      if (is_v) rc = &vchunk;
      slot = is_v ? kKN + *rc % kVN : *rc % kKN;
      use = is_v ? *rc / kVN : *rc / kKN;
    } else {
      slot = chunk % kN;
      use = chunk / kN;
    }
    if (use > 0) mbar_wait(&S.kv_empty[slot], (use - 1) & 1, abort);
    const bool ok = !*abort;
    if (leader && ok) mbar_arrive_expect_tx(&S.kv_full[slot], kChunkBytes);
    load_rows(ring_chunk(S, slot), is_v ? &seq->tmap_v : &seq->tmap_k, C::kBoxDims * c, w, y,
              &S.kv_full[slot], evict_first, ok);
    if (ok) *(rc == &vchunk ? &vissued : &issued) = *rc + 1;
    ++*rc;
  };
  // Q of work item `item` into its buffer (after the previous user of the buffer is done).
  auto issue_q = [&](int item_no, const WorkItem& w) {
    const int qb = item_no % C::kQBufs, qu = item_no / C::kQBufs;
    if (qu > 0) mbar_wait(&S.q_empty[qb], (qu - 1) & 1, abort);
    if (!*abort) {
      if (leader) {
        mbar_arrive_expect_tx(&S.q_full[qb], 4 * kQChunkBytes);
        uint8_t* qd = q_buf<kFp8>(S, qb);
        for (int c = 0; c < 4; ++c)
          tma_load_2d(qd + c * kQChunkBytes, q_map, 64 * c, w.b * kHeads, &S.q_full[qb]);
      }
      q_issued = item_no + 1;
    }
  };
  // In a layer step the K/V rows (and the split plan) were written by kernels that completed
  // before this one launched, so the first boxes of the first item -- a ring-full, which
  // needs no free slot -- stream in while the previous kernel (which writes q) finishes. In a
  // standalone call the CTA has already waited (it built the plan), so the first item's Q,
  // which its first product needs, goes out ahead of the ring.
  int first_done = 0;
  const bool q0_early = !a.plan_early;
  if (has && q0_early) issue_q(0, it);
  if constexpr (kPaged) {
    if (has) {
      fetch_ids(it);
      store_ids(0);
      if (has_nx) fetch_ids(nx);
    }
  }
  if (has) {
    // the boxes that find their slot free: the first kN, or with two rings the leading boxes
    // that are the first use of their ring's slots
    const int total = kBoxesPerTile * num_tiles(it);
    if constexpr (C::kSplitIssue) {
      int nk = 0, nv = 0;
      while (first_done < total) {
        bool is_v;
        int t, c;
        classify(it, first_done, is_v, t, c);
        if (is_v ? nv >= static_cast<int>(kVN) : nk >= static_cast<int>(kKN)) break;
        (is_v ? nv : nk) += 1;
        issue_box(it, first_done++);
      }
    } else {
      first_done = total < static_cast<int>(kN) ? total : static_cast<int>(kN);
      for (int j = 0; j < first_done; ++j) issue_box(it, j);
    }
  }
  pdl_wait();
  while (has) {
    if constexpr (kPaged) {
      if (item > 0) {  // this item's ids, fetched while the previous one streamed
        store_ids(item & 1);
        if (has_nx) fetch_ids(nx);
      }
    }
    if (has_nx && leader) {
      prefetch_tensormap(&a.kv[nx.b].tmap_k);
      prefetch_tensormap(&a.kv[nx.b].tmap_v);
    }
    if (!(item == 0 && q0_early)) issue_q(item, it);
    const int total = kBoxesPerTile * num_tiles(it);
    for (int j = (item == 0 ? first_done : 0); j < total; ++j) issue_box(it, j);
    ++item;
    it = nx;
    has = has_nx;
    if (has) has_nx = plan_get(S.plan, a.batch, cur, nx);
  }
  // Before the CTA may exit, every copy it started must have landed.
  if (*abort) {
    for (uint32_t c = (issued > kKN ? issued - kKN : 0); c < issued; ++c)
      mbar_wait_drain(&S.kv_full[c % kKN], (c / kKN) & 1);
    if constexpr (C::kSplitIssue) {
      for (uint32_t c = (vissued > kVN ? vissued - kVN : 0); c < vissued; ++c)
        mbar_wait_drain(&S.kv_full[kKN + c % kVN], (c / kVN) & 1);
    }
    for (int i = (q_issued > C::kQBufs ? q_issued - C::kQBufs : 0); i < q_issued; ++i)
      mbar_wait_drain(&S.q_full[i % C::kQBufs], (i / C::kQBufs) & 1);
  }
}

// ---------------------------------------------------------------------------------------
// MMA issue (one elected lane issues; the warp runs its loop converged). kRole 0: S and PV
// from one warp (bf16); FP8: kRole 1, the S products (warp 1, K ring), and kRole 2, the PV
// products (warp kPvWarp, V ring).
// ---------------------------------------------------------------------------------------
template <bool kFp8, bool kPaged, int kRole>
__device__ void run_mma(TcSmem& S, const AttnArgs& a, int g, uint32_t tmem, bool leader) {
  using C = Cfg<kFp8>;
  static_assert((kRole == 0) == !C::kSplitIssue, "one issuing warp for bf16, two for FP8");
  constexpr uint32_t kSlots = C::kSlots;
  // FP8 rings: K boxes in slots [0, kKS), V boxes in [kKS, kSlots); each role counts its own
  constexpr uint32_t kKS = C::kKSlots, kVS = kSlots > kKS ? kSlots - kKS : 1;
  constexpr int kC = C::kTileBoxes;
  volatile int* abort = &S.abort_flag;
  const int lane = threadIdx.x & 31;
  constexpr bool paged = kPaged;
  uint32_t chunk = 0;
  uint32_t gt = 0;  // tiles issued so far by this CTA (all items)
  int item = 0;

  plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem& it) {
    const int n = num_tiles(it);
    auto rows_kept = [&](int t) {
      int y, a0, e0;
      tile_window(it, t, paged, y, a0, e0);
      return window_rows_kept(paged, y, e0);
    };
    const int qb = item % C::kQBufs, qu = item / C::kQBufs;
    // FP8: q_ready completes once per item (the split of its Q); the PV role needs no Q
    if (kRole != 2) mbar_wait(kFp8 ? &S.q_ready : &S.q_full[qb], (kFp8 ? item : qu) & 1, abort);
    tc_fence_after();
    const uint32_t q_base = smem_u32(q_buf<kFp8>(S, qb));

    // one MMA: kind::f16 (bf16) or kind::f8f6f4 (e4m3)
    auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
      if constexpr (kFp8)
        umma_f8_ss(d, ad, bd, idesc, acc);
      else
        umma_f16_ss(d, ad, bd, idesc, acc);
    };
    // 128-byte rows: an MMA's K step is 32 bytes of a K-major row, or kMmaK rows (kMmaK / 8
    // swizzle atoms of 1024 bytes) of an MN-major operand
    constexpr int kStepsPerBox = 128 / (C::kMmaK * (kFp8 ? 1 : 2));  // 4
    constexpr uint32_t kMnStep = C::kMmaK / 8 * 1024;
    constexpr int kQStride = kFp8 ? kQ8ChunkBytes : kQChunkBytes;

    auto issue_s = [&](uint32_t tile) {
      const uint32_t j = tile & 1, k = tile >> 1;
      if (k > 0) mbar_wait(&S.s_free[j], (k - 1) & 1, abort);
      tc_fence_after();
      const uint32_t d = tmem + kTmemS + C::kSCols * j;
      if constexpr (kFp8) {
        // K(tile): both boxes, then the 8 MMAs back to back. FP8 tiles are consumed slower
        // than they stream, so the ring runs ahead and the boxes have landed; a wait or a
        // commit between MMAs would stall the issue stream.
        const uint32_t s0 = chunk % kKS, s1 = (chunk + 1) % kKS;
        mbar_wait(&S.kv_full[s0], (chunk / kKS) & 1, abort);
        mbar_wait(&S.kv_full[s1], ((chunk + 1) / kKS) & 1, abort);
        tc_fence_after();
        if (!*abort && leader) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t a_base = smem_u32(ring_chunk(S, c == 0 ? s0 : s1));
#pragma unroll
            for (int kk = 0; kk < kStepsPerBox; ++kk) {
              const uint64_t ad = sdesc_sw128(a_base + 32 * kk, 16, 1024);
              const uint64_t bd = sdesc_sw128(q_base + c * kQStride + 32 * kk, 16, 1024);
              mma(d, ad, bd, C::kIdescS, (c | kk) != 0);
            }
          }
          umma_commit(&S.kv_empty[s0]);
          umma_commit(&S.kv_empty[s1]);
          umma_commit(&S.s_full[j]);
        }
        chunk += 2;
      } else {
        // K(tile): kC ring boxes, each used as soon as TMA has landed it
        for (int c = 0; c < kC; ++c) {
          const uint32_t slot = chunk % kSlots, use = chunk / kSlots;
          mbar_wait(&S.kv_full[slot], use & 1, abort);
          tc_fence_after();
          if (!*abort && leader) {
            const uint32_t a_base = smem_u32(ring_chunk(S, slot));
#pragma unroll
            for (int kk = 0; kk < kStepsPerBox; ++kk) {
              const uint64_t ad = sdesc_sw128(a_base + 32 * kk, 16, 1024);
              const uint64_t bd = sdesc_sw128(q_base + c * kQStride + 32 * kk, 16, 1024);
              mma(d, ad, bd, C::kIdescS, (c | kk) != 0);
            }
            umma_commit(&S.kv_empty[slot]);
          }
          ++chunk;
        }
        if (!*abort && leader) umma_commit(&S.s_full[j]);
      }
    };

    auto issue_pv = [&](uint32_t tile, bool first, int keep) {
      mbar_wait(&S.p_full, tile & 1, abort);
      if (first && item > 0) mbar_wait(&S.o_free, (item - 1) & 1, abort);
      tc_fence_after();
      const uint32_t p_base = smem_u32(S.p);
      if constexpr (kFp8) {
        // V(tile): both boxes (one per half of V^T: 128 dims, one M=128 product each), then
        // the 8 MMAs back to back, as for S
        const uint32_t s0 = kKS + chunk % kVS, s1 = kKS + (chunk + 1) % kVS;
        mbar_wait(&S.kv_full[s0], (chunk / kVS) & 1, abort);
        mbar_wait(&S.kv_full[s1], ((chunk + 1) / kVS) & 1, abort);
        tc_fence_after();
        if (kPaged && keep < kTile && __shfl_sync(0xffffffffu, *abort, 0) == 0) {
          // paged cache, the sequence's last window: V rows past its end are zeroed (see
          // the bf16 branch below)
          zero_chunk_rows(ring_chunk(S, s0), keep, lane);
          zero_chunk_rows(ring_chunk(S, s1), keep, lane);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (!*abort && leader) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t d = tmem + C::kTmemO + C::kSCols * h;
            const uint32_t a_base = smem_u32(ring_chunk(S, h == 0 ? s0 : s1));
#pragma unroll
            for (int kt = 0; kt < kTile / C::kMmaK; ++kt) {
              const uint64_t ad = sdesc_sw128(a_base + kMnStep * kt, kChunkBytes, 1024);
              const uint64_t bd = sdesc_sw128(p_base + kMnStep * kt, kPBytes, 1024);
              mma(d, ad, bd, C::kIdescPV, !(first && kt == 0));
            }
          }
          umma_commit(&S.kv_empty[s0]);
          umma_commit(&S.kv_empty[s1]);
          umma_commit(&S.p_free);
        }
        chunk += 2;
      } else {
        // each half of V^T (the 128 dims of one M=128 product: two bf16 boxes) is used as soon
        // as TMA has landed it
        constexpr int kPerHalf = kC / 2;
        for (int h = 0; h < 2; ++h) {
          const uint32_t c0 = chunk + kPerHalf * h;
          uint32_t sl[kPerHalf];
#pragma unroll
          for (int i = 0; i < kPerHalf; ++i) {
            sl[i] = (c0 + i) % kSlots;
            mbar_wait(&S.kv_full[sl[i]], ((c0 + i) / kSlots) & 1, abort);
          }
          tc_fence_after();
          if (kPaged && keep < kTile && __shfl_sync(0xffffffffu, *abort, 0) == 0) {
            // paged cache, the sequence's last window: V rows past its end may hold any
            // bytes (NaN too) and meet a zero weight, so they are zeroed before PV (the
            // whole warp runs this loop; the abort flag is read once for all its lanes)
#pragma unroll
            for (int i = 0; i < kPerHalf; ++i) zero_chunk_rows(ring_chunk(S, sl[i]), keep, lane);
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (!*abort && leader) {
            const uint32_t d = tmem + C::kTmemO + C::kSCols * h;
            const uint32_t a_base = smem_u32(ring_chunk(S, sl[0]));
#pragma unroll
            for (int kt = 0; kt < kTile / C::kMmaK; ++kt) {
              // bf16: the half's two boxes are adjacent slots, kChunkBytes apart along M
              const uint64_t ad = sdesc_sw128(a_base + kMnStep * kt, kChunkBytes, 1024);
              const uint64_t bd = sdesc_sw128(p_base + kMnStep * kt, kPBytes, 1024);
              mma(d, ad, bd, C::kIdescPV, !(first && kt == 0));
            }
#pragma unroll
            for (int i = 0; i < kPerHalf; ++i) umma_commit(&S.kv_empty[sl[i]]);
          }
        }
        chunk += kC;
        if (!*abort && leader) umma_commit(&S.p_free);
      }
    };

    if constexpr (kRole == 0) {
      for (int t = 0; t < n; ++t) {
        issue_s(gt + t);
        if (t >= 1) issue_pv(gt + t - 1, t - 1 == 0, rows_kept(t - 1));
      }
      if (!*abort && leader) umma_commit(&S.q_empty[qb]);
      issue_pv(gt + n - 1, n == 1, rows_kept(n - 1));
    } else if constexpr (kRole == 1) {
      for (int t = 0; t < n; ++t) issue_s(gt + t);
      if (!*abort && leader) umma_commit(&S.q_empty[qb]);
    } else {
      for (int t = 0; t < n; ++t) issue_pv(gt + t, t == 0, rows_kept(t));
    }
    gt += n;
    ++item;
  });
  // Every MMA issued must be complete before the tensor memory is released.
  if (leader) umma_commit(&S.mma_done);
  mbar_wait_drain(&S.mma_done, 0);
}

// ---------------------------------------------------------------------------------------
// FP8 caches: e4m3 pairs, and the split of Q (run by the eight softmax warps)
// ---------------------------------------------------------------------------------------

// f16x2 -> two e4m3 codes (round to nearest even, saturating at 448), low half -> low byte
__device__ __forceinline__ uint16_t f16x2_to_e4m3x2(uint32_t v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(v));
  return r;
}

// two e4m3 codes -> f16x2 (exact)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// A pair of values (f16x2, |v| <= 256) as e4m3 hi and lo parts: hi = e4m3(v), lo =
// e4m3(v - hi) (v - hi is exact in f16).
__device__ __forceinline__ void split_e4m3x2(uint32_t v, uint16_t& hi, uint16_t& lo) {
  hi = f16x2_to_e4m3x2(v);
  lo = f16x2_to_e4m3x2(hsub2_u32(v, e4m3x2_to_f16x2(hi)));
}

// Q of work item `item` (bf16, four TMA boxes of [64 heads x 64 dims]) -> in place, two
// chunks of [128 rows x 128 dims] e4m3 (row h: the hi part of head h; row 64 + h: its lo
// part; 128-byte swizzle), scaled by 2^-e with e chosen so that the largest |q| maps into
// [128, 256). Returns e. Each of the softmax threads takes kPer consecutive dims of one head:
// kPer / 8 16-byte pieces of one raw box row in, kPer / 16 pieces of the hi row and as many
// of the lo row out. Every thread has read its input before any thread writes: outputs
// overlap inputs. (Not inlined: it runs once per work item, and inlined it pushed the
// softmax loop to spill.)
__device__ __noinline__ int convert_q8(TcSmem& S, int item, int st, int swarp, int lane,
                                      volatile int* abort) {
  using C = Cfg<true>;
  constexpr int kPer = kHeads * kHeadDim / (32 * C::kSoftmaxWarps);  // dims per thread
  constexpr int kParts = kHeadDim / kPer;                             // threads per head
  static_assert(kPer % 16 == 0 && 64 % kPer == 0, "Q split shares");
  const int qb = item & 1;  // two Q buffers
  mbar_wait(&S.q_full[qb], (item >> 1) & 1, abort);
  uint8_t* const qbuf = q_buf<true>(S, qb);
  const int h = st / kParts, d0 = (st % kParts) * kPer;  // head, first dim
  const uint8_t* src = qbuf + (d0 / 64) * kQChunkBytes + h * 128;
  const int rp0 = (d0 % 64) / 8;  // first raw piece of the row
  uint4 v[kPer / 8];
#pragma unroll
  for (int j = 0; j < kPer / 8; ++j)
    v[j] = *reinterpret_cast<const uint4*>(src + (((rp0 + j) ^ (h & 7)) << 4));
  float mx = 0.f;
#pragma unroll
  for (int j = 0; j < kPer / 8; ++j) {
    const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[k] << 16)),
                           fabsf(__uint_as_float(w[k] & 0xFFFF0000u))));
  }
  mx = warp_max_f32(mx);
  if (lane == 0) S.qmax[swarp] = mx;
  named_bar_sync(C::kBarAll, 32 * C::kSoftmaxWarps);  // also: every raw row has been read
  float m = 0.f;
#pragma unroll
  for (int w = 0; w < C::kSoftmaxWarps; ++w) m = fmaxf(m, S.qmax[w]);
  // m * 2^-e in [128, 256); bf16 values times a power of two in [2^-24, 256] are exact in f16.
  // e >= -100 keeps 2^-e finite (a Q whose largest |q| is below 2^-93 is scaled less).
  const int e = (m > 0.f && m <= 3.0e38f) ? max(ilogbf(m) - 7, -100) : 0;
  const float sc = ldexpf(1.f, -e);
  uint32_t hi[kPer / 4], lo[kPer / 4];  // kPer codes each, four per word
#pragma unroll
  for (int j = 0; j < kPer / 8; ++j) {
    const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      uint16_t h0, l0, h1, l1;
      split_e4m3x2(pack_f16x2(__uint_as_float(w[k] << 16) * sc,
                              __uint_as_float(w[k] & 0xFFFF0000u) * sc), h0, l0);
      split_e4m3x2(pack_f16x2(__uint_as_float(w[k + 1] << 16) * sc,
                              __uint_as_float(w[k + 1] & 0xFFFF0000u) * sc), h1, l1);
      hi[2 * j + k / 2] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
      lo[2 * j + k / 2] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
    }
  }
  uint8_t* chunk = qbuf + (d0 / 128) * kQ8ChunkBytes;
  const int op0 = (d0 % 128) / 16;  // first output piece of the rows
#pragma unroll
  for (int j = 0; j < kPer / 16; ++j) {
    const int pj = op0 + j;
    *reinterpret_cast<uint4*>(chunk + h * 128 + ((pj ^ (h & 7)) << 4)) =
        make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
    const int r = 64 + h;
    *reinterpret_cast<uint4*>(chunk + r * 128 + ((pj ^ (r & 7)) << 4)) =
        make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
  }
  fence_proxy_async_smem();
  named_bar_sync(C::kBarAll, 32 * C::kSoftmaxWarps);  // qmax is read before it is reused
  __syncwarp();
  if (lane == 0) mbar_arrive(&S.q_ready);
  return e;
}

// ---------------------------------------------------------------------------------------
// warps 2 ..: softmax, rescale, epilogue (and the FP8 split of Q)
// ---------------------------------------------------------------------------------------
template <bool kFp8, bool kPaged>
__device__ void run_softmax(TcSmem& S, const AttnArgs& a, int g, uint32_t tmem) {
  using C = Cfg<kFp8>;
  constexpr int GH = C::kGroupHeads;  // heads of this thread's group
  volatile int* abort = &S.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int swarp = warp - 2;                // 0 .. kSoftmaxWarps - 1
  const int group = swarp >> 2;              // heads [GH group, GH (group + 1))
  const int st = threadIdx.x - 64;           // 0 .. 32 kSoftmaxWarps - 1
  const int gt_id = st & 127;                // thread within the group
  const uint32_t gbar = 1 + group;           // the group's named barrier
  const int h0 = group * GH;
  const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
  const int row = quad * 32 + lane;          // tile position / O^T row of this thread
  const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
  // the head whose row sum this lane holds after a transpose-sum (see warp_transpose_sum)
  const int sum_head = GH == 32 ? lane : lane >> 1;
  const bool sum_owner = GH == 32 || (lane & 1) == 0;
  const float s_mul0 = a.scale * kLog2e * (kFp8 ? a.k_scale : 1.f);
  const float v_mul = kFp8 ? a.v_scale : 1.f;
  constexpr bool paged = kPaged;
  uint32_t gt = 0;
  int item = 0;
  uint8_t* const p_row = S.p + row * 128;
  // FP8: the next item's Q is split at the end of the current item, before its epilogue, so
  // that the tensor core can start on it while the epilogue runs
  int n_items = 0;
  if constexpr (kFp8) plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem&) { ++n_items; });
  int q_e = 0;  // FP8: the scale exponent of the current item's Q

  plan_for_each_item(S.plan, a.batch, g, [&](const WorkItem& it) {
    const int n = num_tiles(it);
    // this thread's running sums of P over the positions it has held, per head of its group
    // (taken across the 128 positions only once, at the end of the item)
    float lacc[GH];
    float s_mul = s_mul0;
    if constexpr (kFp8) {
      // Q split into e4m3 hi and lo parts scaled by 2^-e, so the scores carry 2^e
      if (item == 0) q_e = convert_q8(S, item, st, swarp, lane, abort);
      s_mul = s_mul0 * ldexpf(1.f, q_e);
    }

    for (int t = 0; t < n; ++t) {
      int y, a0, e0;
      tile_window(it, t, paged, y, a0, e0);
      const uint32_t tile = gt + t, j = tile & 1, k = tile >> 1;
      const int pos = y + row;
      const bool valid = pos >= a0 && pos < e0;
      const bool full = y >= a0 && y + kTile <= e0;  // every position of the window is used

      mbar_wait(&S.s_full[j], k & 1, abort);
      tc_fence_after();
      float s[GH];
      {
        const uint32_t sa = tmem + lane_addr + kTmemS + C::kSCols * j + h0;
        uint32_t sr[GH];
        tmem_ld_cols<GH>(sa, sr);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < GH; ++h) s[h] = __uint_as_float(sr[h]);
        if constexpr (kFp8) {  // plus the lo parts' scores, 64 columns on (16 at a time)
#pragma unroll
          for (int q = 0; q < GH / 16; ++q) {
            uint32_t lr[16];
            tmem_ld_cols<16>(sa + 64 + 16 * q, lr);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h) s[16 * q + h] += __uint_as_float(lr[h]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[j]);

      // s holds the raw products; the scaled score of head h is s[h] * s_mul (log2 units)
      bool need = (t == 0);
      if (!need && valid) {
#pragma unroll
        for (int h = 0; h < GH; ++h) need |= fmaf(s[h], s_mul, -S.m_thr[h0 + h]) > 0.f;
      }
      if (named_bar_or(gbar, kGroupThreads, need)) {
        // exact per-head max of this tile across the 128 positions
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          const float r = warp_max_f32(valid ? s[h] * s_mul : -INFINITY);
          if (lane == 0) S.red[quad][h0 + h] = r;
        }
        named_bar_sync(gbar, kGroupThreads);
        if (gt_id < GH) {
          const int hh = h0 + gt_id;
          const float mt = fmaxf(fmaxf(S.red[0][hh], S.red[1][hh]), fmaxf(S.red[2][hh], S.red[3][hh]));
          const float mo = t == 0 ? -INFINITY : S.m_used[hh];
          const float mn = fmaxf(mo, mt);
          S.alpha[hh] = exp2f(mo - mn);
          S.m_used[hh] = mn;
          S.m_thr[hh] = mn + C::kRescaleThreshold;
          S.m_p[hh] = mn - C::kPExp;
        }
        named_bar_sync(gbar, kGroupThreads);
        if (t == 0) {
#pragma unroll
          for (int h = 0; h < GH; ++h) lacc[h] = 0.f;
        } else {
#pragma unroll
          for (int h = 0; h < GH; ++h) lacc[h] *= S.alpha[h0 + h];
          // O must hold PV(t-1) before it is rescaled
          mbar_wait(&S.p_free, (tile - 1) & 1, abort);
          tc_fence_after();
          // each O^T half (FP8: its hi and its lo columns)
#pragma unroll 1
          // (16 columns at a time: the scores and running sums are live here too)
          for (int hp = 0; hp < (kFp8 ? 4 : 2) * (GH / 16); ++hp) {
            uint32_t o[16];
            const int q = hp % (GH / 16), hq = hp / (GH / 16);
            const uint32_t addr = tmem + lane_addr + C::kTmemO + C::kSCols * (hq & 1) +
                                  64 * (hq >> 1) + h0 + 16 * q;
            tmem_ld_cols<16>(addr, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h)
              o[h] = __float_as_uint(__uint_as_float(o[h]) * S.alpha[h0 + 16 * q + h]);
            tmem_st_cols<16>(addr, o);
          }
          tmem_wait_st();
        }
      }

      // probabilities, rounded to what the tensor core reads (bf16; for FP8 caches e4m3 hi
      // and lo parts), this group's share of the P^T row, and the running sums: of the bf16
      // values, or for FP8 caches of the float32 probabilities (the pair is within 2^-8 of
      // each, and taking it apart again costs the softmax warps, which pace the FP8 tile)
      // The P^T buffer is free once PV(t-1) has read it. Each 16-byte piece of this thread's
      // 128-byte P^T row (positions are rows, 128-byte swizzle) is stored as soon as it is
      // complete: bf16, heads 8 c .. 8 c + 7 in logical piece c; FP8, the hi codes of heads
      // 16 c .. 16 c + 15 in piece c < 4 and their lo codes in piece 4 + c.
      if (tile >= 1) mbar_wait(&S.p_free, (tile - 1) & 1, abort);
      auto prob = [&](int h) {
        const float p = ex2(fmaf(s[h], s_mul, -S.m_p[h0 + h]));
        return (!full && !valid) ? 0.f : p;  // outside the item (also any NaN read there)
      };
      auto store_piece = [&](int cl, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
        *reinterpret_cast<uint4*>(p_row + ((cl ^ (row & 7)) << 4)) = make_uint4(w0, w1, w2, w3);
      };
      if constexpr (kFp8) {
#pragma unroll
        for (int c = 0; c < GH / 16; ++c) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int h = 16 * c + 2 * i;
            const float p0 = prob(h), p1 = prob(h + 1);
            uint16_t hi, lo;
            split_e4m3x2(pack_f16x2(p0, p1), hi, lo);
            if ((i & 1) == 0) {
              hw[i / 2] = hi;
              lw[i / 2] = lo;
            } else {
              hw[i / 2] |= static_cast<uint32_t>(hi) << 16;
              lw[i / 2] |= static_cast<uint32_t>(lo) << 16;
            }
            lacc[h] += p0;
            lacc[h + 1] += p1;
          }
          store_piece(group * (GH / 16) + c, hw[0], hw[1], hw[2], hw[3]);
          store_piece(4 + group * (GH / 16) + c, lw[0], lw[1], lw[2], lw[3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < GH / 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int h = 8 * c + 2 * i;
            w[i] = pack_bf16x2(prob(h), prob(h + 1));
            lacc[h] += __uint_as_float(w[i] << 16);
            lacc[h + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
          }
          store_piece(group * (GH / 8) + c, w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full);
    }
    gt += n;
    if constexpr (kFp8) {
      // every S of this item has completed (its scores were read above), and the next Q
      // sits in the other buffer
      if (item + 1 < n_items) q_e = convert_q8(S, item + 1, st, swarp, lane, abort);
    }

    // ---- epilogue of the item (each group for its heads) ----
    const float lsum_w = warp_transpose_sum<GH>(lacc, lane);  // this warp's positions
    if (sum_owner) S.red[quad][h0 + sum_head] = lsum_w;
    named_bar_sync(gbar, kGroupThreads);
    if (gt_id < GH) {
      const int hh = h0 + gt_id;
      S.lsum[hh] = S.red[0][hh] + S.red[1][hh] + S.red[2][hh] + S.red[3][hh];
    }
    // O^T holds PV of the last tile once its commit has landed
    mbar_wait(&S.p_free, (gt - 1) & 1, abort);
    tc_fence_after();
    // one decision for the whole group, so that all its threads take the same barriers
    const bool ok = !named_bar_or(gbar, kGroupThreads, *abort != 0);
    uint16_t* out = a.out + (size_t)it.b * kQWidth;
    float* pacc = it.slot >= 0 ? partial_acc(a.partials, it.slot) : nullptr;
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t o[GH];
      const uint32_t oa = tmem + lane_addr + C::kTmemO + C::kSCols * hf + h0;
      tmem_ld_cols<GH>(oa, o);
      tmem_wait_ld();
      if constexpr (kFp8) {  // O = (V . P_hi) + (V . P_lo), the lo columns 16 at a time
#pragma unroll
        for (int q = 0; q < GH / 16; ++q) {
          uint32_t ol[16];
          tmem_ld_cols<16>(oa + 64 + 16 * q, ol);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 16; ++h)
            o[16 * q + h] = __float_as_uint(__uint_as_float(o[16 * q + h]) + __uint_as_float(ol[h]));
        }
      }
      const int d = hf * 128 + row;
      if (ok) {
        if (it.slot < 0) {
#pragma unroll
          for (int h = 0; h < GH; ++h)
            out[(h0 + h) * kHeadDim + d] =
                f32_to_bf16_bits(__uint_as_float(o[h]) * (v_mul / S.lsum[h0 + h]));
        } else {
#pragma unroll
          for (int h = 0; h < GH; ++h) pacc[(h0 + h) * kHeadDim + d] = __uint_as_float(o[h]);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.o_free);

    if (it.slot >= 0 && ok && gt_id < GH) {
      partial_m(a.partials, it.slot)[h0 + gt_id] = S.m_used[h0 + gt_id];
      partial_l(a.partials, it.slot)[h0 + gt_id] = S.lsum[h0 + gt_id];
    }
    // m_used / lsum / red of this group's heads are rewritten by the next item only after
    // the group's next barrier
    ++item;
  });
}

template <bool kFp8, bool kPaged>
__global__ void __launch_bounds__(Cfg<kFp8>::kBoundThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap q_map, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < Cfg<kFp8>::kSlots; ++i) {
      mbar_init(&S.kv_full[i], 1);
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.q_full[i], 1);
      mbar_init(&S.q_empty[i], 1);
    }
    mbar_init(&S.q_ready, Cfg<kFp8>::kSoftmaxWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], Cfg<kFp8>::kSoftmaxWarps);
    }
    mbar_init(&S.p_full, Cfg<kFp8>::kSoftmaxWarps);
    mbar_init(&S.p_free, 1);
    mbar_init(&S.o_free, Cfg<kFp8>::kSoftmaxWarps);
    mbar_init(&S.mma_done, Cfg<kFp8>::kMmaWarps);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, Cfg<kFp8>::kTmemCols);
    tmem_relinquish();
  }
  pdl_launch_dependents();  // the combine kernel may start launching; it waits for us
  if (!a.plan_early && threadIdx.x == 0 && a.batch > 0) {
    // The tensor maps of the sequence this CTA most likely starts in (where it would with
    // equal lengths), fetched while the plan is built; the KV table is written only by the
    // host-side table set-up, never by a kernel, so this needs no wait.
    const KvSeq* kv = a.kv + min(a.batch - 1, static_cast<int>((int64_t)g * a.batch / gridDim.x));
    prefetch_tensormap(&kv->tmap_k);
    prefetch_tensormap(&kv->tmap_v);
  }
  if (a.plan_early) {
    // the split plan, computed during the layer step's x-projection by an extra block of
    // the x-projection's finish kernel
    plan_load(S.plan, a.plan, a.batch);
  } else {
    // a standalone call: every CTA builds the (small) plan on chip once seq_lens are final;
    // CTA 0 reports rejected lengths and writes the combine's per-sequence split info
    pdl_wait();
    plan_build(S.plan, a.seq_lens, a.kv, a.batch, a.grid, a.err, g == 0);
    if (g == 0) write_seq_info(S.plan, a.seq_info, a.batch);
  }
  // This kernel was picked for the layout the caller stated; a table of the other layout
  // gets no attention (an empty plan) and an error bit.
  if (threadIdx.x == 0 && (S.plan.page_size != 0) != kPaged) {
    S.plan.grid = 0;
    atomicOr(a.err, kErrLayout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    run_producer<kFp8, kPaged>(S, &q_map, a, g, lane == 0);
  } else if (warp == 1) {
    run_mma<kFp8, kPaged, Cfg<kFp8>::kSplitIssue ? 1 : 0>(S, a, g, tmem, lane == 0);
  } else {
    bool pv_warp = false;
    if constexpr (Cfg<kFp8>::kSplitIssue) {
      if (warp == Cfg<kFp8>::kPvWarp) {
        run_mma<kFp8, kPaged, 2>(S, a, g, tmem, lane == 0);
        pv_warp = true;
      }
    }
    if (!pv_warp) run_softmax<kFp8, kPaged>(S, a, g, tmem);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && S.abort_flag) atomicOr(a.err, kErrTimeout);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, Cfg<kFp8>::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// combine: one block per (sequence, group of 4 heads); each thread owns kHT of the 4 heads
// and two dims, so a block has 4 / kHT * 128 threads.
//   M[h] = max_i m_i[h],  L[h] = sum_i l_i[h] 2^(m_i[h] - M[h]),
//   out[h][d] = v_mul / L[h] * sum_i 2^(m_i[h] - M[h]) acc_i[h][d].
// Up to kOnePass(kHT) splits, every split's m, l and accumulators are loaded at once (one
// round trip to L2); beyond that the weights go through shared memory first. Two shapes:
// kHT = 2 (256 threads) for batches of few long sequences, which split many ways and need
// their merge in one round trip; kHT = 4 (128 threads, fewer registers per block) for large
// batches, whose many blocks must fit the SMs at once. Sequences finished by a single work
// item were written by the attention kernel; rejected sequences (no split) get a zero
// output here.
// ---------------------------------------------------------------------------------------
constexpr int kCombineHeads = 4;
constexpr int kCombineMaxSplits = kMaxAttnGrid;  // a sequence has at most grid splits

template <int kHT>
struct CombineCfg {
  static constexpr int kThreads = kCombineHeads / kHT * 128;
  static constexpr int kOnePass = kHT == 2 ? 6 : 3;
  static constexpr int kMinBlocks = kHT == 2 ? 4 : 8;
};

template <int kHT>
__global__ void __launch_bounds__(CombineCfg<kHT>::kThreads, CombineCfg<kHT>::kMinBlocks)
    attention_combine_kernel(AttnArgs a) {
  using C = CombineCfg<kHT>;
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x, h0 = blockIdx.y * kCombineHeads, tid = threadIdx.x;
  const int2 info = a.seq_info[b];
  const int base = info.x, ns = info.y;
  uint32_t* out = reinterpret_cast<uint32_t*>(a.out + (size_t)b * kQWidth + h0 * kHeadDim);
  if (ns == 0) {
    for (int i = tid; i < kCombineHeads * kHeadDim / 2; i += C::kThreads) out[i] = 0u;
    return;
  }
  if (ns == 1) return;
  const float v_mul = a.kv_dtype == MFA_KV_FP8_E4M3 ? a.v_scale : 1.f;
  const int hg = tid >> 7, hl = h0 + kHT * hg;  // this thread's first head
  const int d2 = tid & 127;                     // dims 2 d2, 2 d2 + 1
  uint32_t* o_out = out + (kHT * hg) * kHeadDim / 2 + d2;
  auto head_of = [](const float4& v, int h) { return h == 0 ? v.x : h == 1 ? v.y : h == 2 ? v.z : v.w; };
  auto ld_heads = [&](const float* p) {  // kHT consecutive floats from head hl on
    if constexpr (kHT == 4) return __ldcg(reinterpret_cast<const float4*>(p + hl));
    const float2 v = __ldcg(reinterpret_cast<const float2*>(p + hl));
    return make_float4(v.x, v.y, 0.f, 0.f);
  };
  if (ns <= C::kOnePass) {
    float4 mv[C::kOnePass], lv[C::kOnePass];
    float2 xv[C::kOnePass][kHT];
#pragma unroll
    for (int i = 0; i < C::kOnePass; ++i) {
      if (i < ns) {
        mv[i] = ld_heads(partial_m(a.partials, base + i));
        lv[i] = ld_heads(partial_l(a.partials, base + i));
        const float* acc = partial_acc(a.partials, base + i) + hl * kHeadDim + 2 * d2;
#pragma unroll
        for (int h = 0; h < kHT; ++h)
          xv[i][h] = __ldcg(reinterpret_cast<const float2*>(acc + h * kHeadDim));
      }
    }
#pragma unroll
    for (int h = 0; h < kHT; ++h) {
      float M = -INFINITY;
#pragma unroll
      for (int i = 0; i < C::kOnePass; ++i)
        if (i < ns) M = fmaxf(M, head_of(mv[i], h));
      float L = 0.f;
      float2 o = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < C::kOnePass; ++i) {
        if (i < ns) {
          const float w = exp2f(head_of(mv[i], h) - M);
          L = fmaf(head_of(lv[i], h), w, L);
          o.x = fmaf(w, xv[i][h].x, o.x);
          o.y = fmaf(w, xv[i][h].y, o.y);
        }
      }
      const float inv = v_mul / L;
      o_out[h * kHeadDim / 2] = pack_bf16x2(o.x * inv, o.y * inv);
    }
    return;
  }
  // More splits: (1) every (split, head) pair's m and l in one round trip; (2) the weights
  // v_mul 2^(m_i - M) / L per head, one warp per head; (3) the accumulators, whose loads
  // no longer depend on any arithmetic, so many splits stay in flight.
  __shared__ float sm[kCombineHeads][kCombineMaxSplits];
  __shared__ float sl[kCombineHeads][kCombineMaxSplits];
  for (int t = tid; t < kCombineHeads * ns; t += C::kThreads) {
    const int i = t >> 2, h = t & 3;
    sm[h][i] = __ldcg(partial_m(a.partials, base + i) + h0 + h);
    sl[h][i] = __ldcg(partial_l(a.partials, base + i) + h0 + h);
  }
  __syncthreads();
  if (tid < 32 * kCombineHeads) {
    const int h = tid >> 5, lane = tid & 31;  // warp h: head h0 + h
    float mx = -INFINITY;
    for (int i = lane; i < ns; i += 32) mx = fmaxf(mx, sm[h][i]);
    mx = warp_max_f32(mx);
    float ls = 0.f;
    for (int i = lane; i < ns; i += 32) ls = fmaf(sl[h][i], exp2f(sm[h][i] - mx), ls);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    __syncwarp();
    const float sc = v_mul / ls;
    for (int i = lane; i < ns; i += 32) sl[h][i] = sc * exp2f(sm[h][i] - mx);  // weights
  }
  __syncthreads();
  float2 o[kHT];
#pragma unroll
  for (int h = 0; h < kHT; ++h) o[h] = make_float2(0.f, 0.f);
#pragma unroll 8
  for (int i = 0; i < ns; ++i) {
    const float* acc = partial_acc(a.partials, base + i) + hl * kHeadDim + 2 * d2;
#pragma unroll
    for (int h = 0; h < kHT; ++h) {
      const float2 x = __ldcg(reinterpret_cast<const float2*>(acc + h * kHeadDim));
      const float w = sl[kHT * hg + h][i];
      o[h].x = fmaf(w, x.x, o[h].x);
      o[h].y = fmaf(w, x.y, o[h].y);
    }
  }
#pragma unroll
  for (int h = 0; h < kHT; ++h) o_out[h * kHeadDim / 2] = pack_bf16x2(o[h].x, o[h].y);
}

}  // namespace

cudaError_t launch_attention_combine(const AttnArgs& a, cudaStream_t s) {
  // large batches split each sequence a few ways over the grid: many small merges, blocks
  // with fewer registers so they all fit at once; small batches: few long sequences split
  // many ways, each merge in one round trip
  const dim3 grid(a.batch, kHeads / kCombineHeads, 1);
  if (a.batch >= 64)
    return launch_pdl(attention_combine_kernel<4>, grid, dim3(CombineCfg<4>::kThreads), 0, s, a);
  return launch_pdl(attention_combine_kernel<2>, grid, dim3(CombineCfg<2>::kThreads), 0, s, a);
}

size_t attention_tc_smem_bytes() { return sizeof(TcSmem) + 1024; }

template <bool kFp8, bool kPaged>
static cudaError_t launch_tc(const CUtensorMap& q_map, const AttnArgs& a, cudaStream_t s) {
  const size_t smem = attention_tc_smem_bytes();
  static std::atomic<uint64_t> smem_set{0};
  if (!set_smem_limit_once(reinterpret_cast<const void*>(attention_tc_kernel<kFp8, kPaged>),
                           (int)smem, &smem_set))
    return cudaErrorInvalidValue;
  return launch_pdl(attention_tc_kernel<kFp8, kPaged>, dim3(a.grid), dim3(Cfg<kFp8>::kThreads), smem, s,
                    q_map, a);
}

// Contiguous and paged caches have kernels of their own (the caller's description picks
// one): a paged window never slides, and page lookups would slow the contiguous loop.
cudaError_t launch_attention_tc(const CUtensorMap& q_map, const AttnArgs& a, cudaStream_t s) {
  const bool fp8 = a.kv_dtype == MFA_KV_FP8_E4M3;
  if (a.page_size != 0)
    return fp8 ? launch_tc<true, true>(q_map, a, s) : launch_tc<false, true>(q_map, a, s);
  return fp8 ? launch_tc<true, false>(q_map, a, s) : launch_tc<false, false>(q_map, a, s);
}

}  // namespace mfa
