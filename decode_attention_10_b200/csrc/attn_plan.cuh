// Length-aware split plan of the decode attention. In a layer step one extra block of the
// x-projection's finish kernel builds it (it needs only seq_lens and the KV table) and
// stores it for the attention CTAs; a standalone attention call builds it on chip in every
// attention CTA.
//
// The cached positions of all sequences are cut into tiles of kTile positions and laid end
// to end (sequence 0's tiles, then sequence 1's, ...). CTA g of a persistent grid of G CTAs
// (G capped at the tile count NT, so that no CTA of the plan is empty)
// takes the contiguous tile range [bound(g), bound(g + 1)), bound(g) = floor(g * NT / G),
// so every CTA streams the same number of KV bytes (to within one tile) whatever the mix
// of lengths. The part of one sequence that falls in one CTA's range is a work item. A
// sequence covered by a single CTA is finished in place; a sequence split over n > 1 CTAs
// gets n partial slots (m, l, acc), which the combine kernel merges.
#pragma once

#include "mfa_internal.cuh"

namespace mfa {

struct PlanSmem {
  int32_t tile_start[kMaxBatch + 1];  // exclusive prefix of tiles per sequence
  int32_t slot_base[kMaxBatch];       // exclusive prefix of partial slots per sequence
  int32_t len[kMaxBatch];             // attended positions (0 for rejected sequences)
  int32_t grid;  // CTAs that get work: min(G, total tiles), so none of them is empty
  int32_t flag;
  int32_t page_size;  // the KV table's layout: 0 contiguous, else rows per page
};

// The products below stay under 2^27 (NT <= kMaxBatch * kMaxTilesPerSeq = 2^19 tiles, G <=
// kMaxAttnGrid = 2^8), so 32-bit unsigned arithmetic computes them exactly (a 64-bit division
// is a long software routine on the GPU, and the plan is on the critical path of every call).
constexpr uint32_t kMaxTilesPerSeq = (MFA_MAX_CONTEXT + kTile - 1) / kTile;
static_assert(static_cast<uint64_t>(kMaxBatch) * kMaxTilesPerSeq * kMaxAttnGrid < (1ull << 32),
              "plan arithmetic fits 32 bits");

__device__ __forceinline__ int plan_bound(int g, int G, int NT) {
  return static_cast<int>(static_cast<uint32_t>(g) * static_cast<uint32_t>(NT) /
                          static_cast<uint32_t>(G));
}

// CTA owning tile t: the largest g with plan_bound(g) <= t.
__device__ __forceinline__ int plan_cta_of(int t, int G, int NT) {
  return static_cast<int>((static_cast<uint32_t>(t + 1) * static_cast<uint32_t>(G) - 1u) /
                          static_cast<uint32_t>(NT));
}

// Inclusive sum over the lanes of a warp (lane l gets the sum of lanes 0..l).
__device__ __forceinline__ int warp_inclusive_sum(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Build the plan for `batch` sequences over a grid of G CTAs. Lengths outside
// [1, capacity] are rejected (length 0; the output is zero-filled) and, if `report`, flagged.
// Every thread of the block calls it. The lengths are read by all threads at once (one
// round trip to memory); warp 0 then scans the tile counts and the split slots, each lane
// over a contiguous run of sequences, so the block meets at two barriers only.
__device__ inline void plan_build(PlanSmem& P, const int32_t* __restrict__ seq_lens,
                                  const KvSeq* __restrict__ kv, int batch, int G,
                                  uint32_t* err, bool report) {
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    const int L = seq_lens[b];
    const int cap = kv[b].capacity;
    int len = L;
    if (L <= 0) {
      len = 0;
      if (report) atomicOr(err, kErrEmpty);
    } else if (L > cap) {
      len = 0;
      if (report) atomicOr(err, kErrCapacity);
    }
    P.len[b] = len;
    P.tile_start[b] = (len + kTile - 1) / kTile;  // the tile count; scanned below
  }
  if (threadIdx.x == 0) P.page_size = kv[0].page_size;  // the same in every entry
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (batch + 31) / 32;
    const int b0 = min(batch, lane * per), b1 = min(batch, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) sum += P.tile_start[b];
    int incl = warp_inclusive_sum(sum, lane);
    const int NT = __shfl_sync(0xffffffffu, incl, 31);
    int run = incl - sum;
    for (int b = b0; b < b1; ++b) {
      const int n = P.tile_start[b];
      P.tile_start[b] = run;
      run += n;
    }
    const int Ge = min(G, NT);  // CTAs that get work, so none of them is empty
    if (lane == 0) {
      P.tile_start[batch] = NT;
      P.grid = Ge;
    }
    __syncwarp();
    // partial slots: a sequence whose tiles fall in n > 1 CTAs' ranges gets n of them
    sum = 0;
    for (int b = b0; b < b1; ++b) {
      const int ts = P.tile_start[b], te = P.tile_start[b + 1];
      int slots = 0;
      if (te > ts) {
        const int n = plan_cta_of(te - 1, Ge, NT) - plan_cta_of(ts, Ge, NT) + 1;
        slots = n > 1 ? n : 0;
      }
      P.slot_base[b] = slots;
      sum += slots;
    }
    incl = warp_inclusive_sum(sum, lane);
    run = incl - sum;
    for (int b = b0; b < b1; ++b) {
      const int n = P.slot_base[b];
      P.slot_base[b] = run;
      run += n;
    }
  }
  __syncthreads();
}

// The plan in global memory: tile_start[batch + 1], slot_base[batch], len[batch], grid,
// page_size, at fixed offsets of a kPlanBytes buffer.
__device__ inline void plan_store(const PlanSmem& P, int32_t* g, int batch) {
  for (int i = threadIdx.x; i <= batch; i += blockDim.x) g[i] = P.tile_start[i];
  for (int i = threadIdx.x; i < batch; i += blockDim.x) {
    g[kMaxBatch + 1 + i] = P.slot_base[i];
    g[2 * kMaxBatch + 1 + i] = P.len[i];
  }
  if (threadIdx.x == 0) {
    g[3 * kMaxBatch + 1] = P.grid;
    g[3 * kMaxBatch + 2] = P.page_size;
  }
}

__device__ inline void plan_load(PlanSmem& P, const int32_t* __restrict__ g, int batch) {
  for (int i = threadIdx.x; i <= batch; i += blockDim.x) P.tile_start[i] = g[i];
  for (int i = threadIdx.x; i < batch; i += blockDim.x) {
    P.slot_base[i] = g[kMaxBatch + 1 + i];
    P.len[i] = g[2 * kMaxBatch + 1 + i];
  }
  if (threadIdx.x == 0) {
    P.grid = g[3 * kMaxBatch + 1];
    P.page_size = g[3 * kMaxBatch + 2];
  }
}

// Per sequence: its first partial slot and the number of CTAs it is split over (0 for a
// rejected sequence), for the combine kernel.
__device__ inline void write_seq_info(const PlanSmem& P, int2* seq_info, int batch) {
  const int NT = P.tile_start[batch], G = P.grid;
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    const int ts = P.tile_start[b], te = P.tile_start[b + 1];
    const int ns = te > ts ? plan_cta_of(te - 1, G, NT) - plan_cta_of(ts, G, NT) + 1 : 0;
    seq_info[b] = make_int2(P.slot_base[b], ns);
  }
}

struct WorkItem {
  int b;        // sequence
  int tok0;     // first cached position of the item
  int tok1;     // one past the last
  int slot;     // partial slot, or -1 if the sequence is finished by this item alone
  int nsplit;   // CTAs sharing the sequence
  int split;    // this item's index among them (its slot is slot_base[b] + split)
};

// Walk over the work items of CTA g, in order: begin, then get until it returns false.
struct PlanCursor {
  int b;   // next sequence to look at
  int t0;  // the CTA's tile range [t0, t1)
  int t1;
  int g;   // the CTA
};

__device__ inline PlanCursor plan_begin(const PlanSmem& P, int batch, int g) {
  PlanCursor c{batch, 0, 0, g};
  const int NT = P.tile_start[batch];
  const int G = P.grid;
  if (NT == 0 || g >= G) return c;
  c.t0 = plan_bound(g, G, NT);
  c.t1 = plan_bound(g + 1, G, NT);
  // largest b with tile_start[b] <= t0 (that sequence contains tile t0)
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.tile_start[mid] <= c.t0) lo = mid; else hi = mid - 1;
  }
  c.b = lo;
  return c;
}

__device__ inline bool plan_get(const PlanSmem& P, int batch, PlanCursor& c, WorkItem& it) {
  const int NT = P.tile_start[batch];
  const int G = P.grid;
  for (; c.b < batch && P.tile_start[c.b] < c.t1; ++c.b) {
    const int b = c.b;
    const int ts = P.tile_start[b], te = P.tile_start[b + 1];
    if (te <= c.t0 || te == ts) continue;
    const int a0 = max(ts, c.t0), a1 = min(te, c.t1);
    it.b = b;
    it.tok0 = (a0 - ts) * kTile;
    it.tok1 = min(P.len[b], (a1 - ts) * kTile);
    const int gf = plan_cta_of(ts, G, NT);
    it.nsplit = plan_cta_of(te - 1, G, NT) - gf + 1;
    it.split = c.g - gf;
    it.slot = it.nsplit > 1 ? P.slot_base[b] + it.split : -1;
    ++c.b;
    return true;
  }
  return false;
}

// Call f(item) for every work item of CTA g, in order.
template <class F>
__device__ inline void plan_for_each_item(const PlanSmem& P, int batch, int g, F&& f) {
  PlanCursor c = plan_begin(P, batch, g);
  WorkItem it;
  while (plan_get(P, batch, c, it)) f(it);
}

// Partial slot views.
__device__ __forceinline__ float* partial_m(float* base, int slot) {
  return base + (size_t)slot * kPartialFloats;
}
__device__ __forceinline__ float* partial_l(float* base, int slot) {
  return base + (size_t)slot * kPartialFloats + kHeads;
}
__device__ __forceinline__ float* partial_acc(float* base, int slot) {
  return base + (size_t)slot * kPartialFloats + 2 * kHeads;
}

}  // namespace mfa
