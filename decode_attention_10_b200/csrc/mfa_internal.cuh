// Internal definitions shared by the kernels and the C-ABI layer of libmfa.
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver is reached through the runtime)
#include <cuda_runtime.h>

#include <atomic>
#include <stddef.h>
#include <stdint.h>

#include "../../include/mfa.h"

namespace mfa {

// Layer dimensions (Step-3 pages: bud-325 "Key claims"/"Method", redeep architecture table).
constexpr int kHidden = MFA_HIDDEN;     // 7168
constexpr int kRank = MFA_Q_RANK;       // 2048
constexpr int kHeads = MFA_N_HEADS;     // 64
constexpr int kHeadDim = MFA_HEAD_DIM;  // 256
constexpr int kQWidth = kHeads * kHeadDim;  // 16384
constexpr int kMaxBatch = MFA_MAX_BATCH;

// Columns of the hidden-state projection x [W_qdown | W_k | W_v]: 2048 + 256 + 256.
constexpr int kXProjCols = kRank + 2 * kHeadDim;  // 2560
constexpr int kXProjSplits = 7;                   // split-K of the 7168-long reduction
constexpr int kXProjKPerSplit = kHidden / kXProjSplits;  // 1024
static_assert(kHidden % kXProjSplits == 0, "split-K must divide the hidden width");

// Output projection out [B, 16384] -> y [B, 7168]: split-K of the 16384-long reduction
// (56 tiles of 128 features x 2 splits = 112 CTAs).
constexpr int kOProjSplits = 2;
constexpr int kOProjKPerSplit = kQWidth / kOProjSplits;  // 8192

// Attention work unit: the plan hands out whole tiles of this many cached positions.
constexpr int kTile = 128;

// Device-side error bits kept in the workspace header.
enum : uint32_t { kErrCapacity = 1u, kErrEmpty = 2u, kErrTimeout = 4u, kErrLayout = 8u };

// One entry of the device KV table. Contiguous caches: TMA tensor maps of the sequence's own
// K and V rows ([capacity, 256] elements, row-major), their base pointers, page_size 0.
// Paged caches: the maps cover the whole pools ([num_pages, page_size, 256]), k / v are the
// pool bases, and row j of the sequence is row j % page_size of page pages[j / page_size];
// capacity = (pages given to the sequence) * page_size. Every entry of one table has the
// same layout.
struct alignas(128) KvSeq {
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  void* k;
  void* v;
  int32_t capacity;
  int32_t page_size;      // 0: contiguous
  const int32_t* pages;   // paged: this sequence's row of the page table (device)
  int32_t num_pages;      // paged: pages in each pool
  int32_t reserved[23];
};
static_assert(sizeof(KvSeq) == 384, "KvSeq layout");

// The element row, in its K or V buffer (or pool), of cache row `row` of sequence s: the
// sequence's own row, or for a paged cache row % page_size of page pages[row / page_size].
// -1 if the row is outside the sequence's capacity or its page outside the pool.
__device__ inline long long kv_row_index(const KvSeq& s, int row) {
  if (row < 0 || row >= s.capacity) return -1;
  if (s.page_size == 0) return row;
  const int page = s.pages[row / s.page_size];
  if (page < 0 || page >= s.num_pages) return -1;
  return static_cast<long long>(page) * s.page_size + row % s.page_size;
}

// Paged caches: rows per TMA box (a 128-position window is 128 / box rows boxes, each
// inside one page).
__host__ __device__ inline int paged_box_rows(int page_size) {
  return page_size % 128 == 0 ? 128 : 64;
}

// Split-K partial of one attention work item: running max m (log2 domain) and sum l per
// head, and the unnormalized accumulator acc[head][dim], all fp32.
constexpr int kPartialFloats = kHeads + kHeads + kHeads * kHeadDim;  // 16512
constexpr size_t kPartialBytes = kPartialFloats * sizeof(float);     // 66048 = 258 * 256

// Bytes of the attention split plan kept in the workspace (tile_start[kMaxBatch + 1],
// slot_base[kMaxBatch], len[kMaxBatch], grid, page_size).
constexpr size_t kPlanBytes = sizeof(int32_t) * (3 * kMaxBatch + 3);

struct WsLayout {
  size_t err;          // uint32 error bits
  size_t seq_info;     // int2 [kMaxBatch]: (first partial slot, splits) per sequence
  size_t plan;         // the attention split plan (written by the finish kernel's plan block)
  size_t attn_part;    // partial slots
  size_t xproj_part;   // fp32 [kXProjSplits][batch][kXProjCols]
  size_t c_hat;        // bf16 [batch][kRank]
  size_t oproj_part;   // fp32 [kOProjSplits][batch][kHidden]
  size_t x8, x8_scale;        // FP8 path: x as e4m3 [batch][7168] + scales [batch][56]
  size_t chat8, chat8_scale;  // FP8 path: c_hat as e4m3 [batch][2048] + scales [batch][16]
  size_t total;
  int attn_slots;
  int attn_grid;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Persistent attention grid: one CTA per SM, at most kMaxAttnGrid (the combine kernel merges
// at most that many splits of one sequence).
constexpr int kMaxAttnGrid = 256;
inline int attn_grid_for(int num_sms) { return num_sms < kMaxAttnGrid ? num_sms : kMaxAttnGrid; }

inline WsLayout ws_layout(int batch, int num_sms) {
  WsLayout L{};
  size_t off = 0;
  L.err = off;
  off += 256;
  L.seq_info = off;
  off = align_up(off + 2 * sizeof(int32_t) * kMaxBatch, 256);
  L.plan = off;
  off = align_up(off + kPlanBytes, 256);
  L.attn_grid = attn_grid_for(num_sms);
  L.attn_slots = L.attn_grid + batch;  // sum over sequences of their splits <= grid + batch
  L.attn_part = off;
  off = align_up(off + kPartialBytes * (size_t)L.attn_slots, 256);
  L.xproj_part = off;
  off = align_up(off + sizeof(float) * kXProjSplits * (size_t)batch * kXProjCols, 256);
  L.c_hat = off;
  off = align_up(off + sizeof(uint16_t) * (size_t)batch * kRank, 256);
  L.oproj_part = off;
  off = align_up(off + sizeof(float) * kOProjSplits * (size_t)batch * kHidden, 256);
  L.x8 = off;
  off = align_up(off + (size_t)batch * kHidden, 256);
  L.x8_scale = off;
  off = align_up(off + sizeof(float) * (size_t)batch * (kHidden / 128), 256);
  L.chat8 = off;
  off = align_up(off + (size_t)batch * kRank, 256);
  L.chat8_scale = off;
  off = align_up(off + sizeof(float) * (size_t)batch * (kRank / 128), 256);
  L.total = off;
  return L;
}

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel on the stream is still running; it does its own set-up (barriers, TMEM, tensor-map
// prefetch, the attention split plan) and then executes griddepcontrol.wait before it reads
// anything the previous kernels of the step write. Every kernel of the step waits before it
// triggers its own dependents, so "previous kernel complete" is transitive along the stream.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files); all return cudaGetLastError().
// ---------------------------------------------------------------------------------------

// Weight-streaming GEMM on the tensor cores: out^T[n, b] = sum_k W[k, n] X[b, k] for 128
// output features per CTA (grid.x), a range of k per CTA (grid.y: split-K), and up to 256
// rows of X per CTA (grid.z).
struct WGemmArgs {
  int batch;            // rows of X
  int tile_begin;       // first 128-feature tile (of the concatenated outputs)
  int three_weights;    // 1: tiles [0, w0_tiles) read w[0], then w1_tiles of w[1], then w[2]
  int w0_tiles, w1_tiles;
  int kblocks_per_cta;  // 128-wide k blocks per CTA
  float* out_f32;       // fp32 split partials [grid.y][batch][out_ld], or null
  uint16_t* out_bf16;   // bf16 [batch][out_ld] (when out_f32 is null)
  int out_ld;
  uint32_t* err;
  // block-FP8 weights: per weight its scales [N_out / 128][wscale_ld] (row-major, one per
  // 128 x 128 block); null = bf16 weights
  const float* wscale[3];
  int wscale_ld[3];
  // FP8 path: X is e4m3 codes [batch, K] with scales [batch][xscale_ld] (one per 128 k)
  const float* xscale;
  int xscale_ld;
  int n_box, stages, tmem_cols, dbufs;  // filled in by launch_wgemm
};
// w: 3 tensor maps over row-major [K, N_out] bf16 weights, boxes [128 k x 64 features], or
// for block-FP8 weights over [N_out, K] e4m3 codes, boxes [128 features x 128 k];
// xmap over X [batch, K] bf16, boxes [wgemm_n_box(batch) x 64 k]; all with 128-byte swizzle.
// kblocks_per_cta counts blocks of 128 k.
cudaError_t launch_wgemm(const CUtensorMap* w, const CUtensorMap& xmap, WGemmArgs p,
                         int m_tiles, int splits, cudaStream_t s);
int wgemm_n_box(int batch);
int wgemm_n_box_fp8(int batch);  // the FP8 path's X box rows (at most 128 rows per CTA)

struct FinishArgs {
  const float* part;  // x-projection partials
  int batch;
  // query half: c_hat = bf16(rmsnorm(c) * gamma)
  const uint16_t* gamma;  // null = skip the query half
  float eps;
  uint16_t* c_hat;  // [batch, 2048]
  uint8_t* chat8;        // FP8 path: c_hat also as e4m3 [batch, 2048] (null = bf16 path)
  float* chat8_scale;    // FP8 path: its scales [batch, 16], one per 128 columns
  // K/V half: append bf16 / e4m3 rows
  const KvSeq* kv;  // null = skip the K/V half
  int kv_dtype;
  float k_scale, v_scale;
  const int32_t* pos;      // device [batch]: row to write
  int pos_from_len;        // 1: row = pos[b] - 1 (pos holds seq_lens)
  uint32_t* err;
  // the attention's split plan (layer step): one extra block builds it from pos (= seq_lens)
  // and the KV table while the x-projection runs, and stores it with the combine's
  // per-sequence info; null = no plan block
  int32_t* plan;
  int2* seq_info;
  int attn_grid;
};
cudaError_t launch_xproj_finish(const FinishArgs& a, cudaStream_t s);

// The FP8 path's activations: a [rows, k] bf16 -> e4m3 codes [rows, k] and float32 scales
// [rows, k / 128], per row and group of 128 values (query_path.cu).
cudaError_t launch_quantize_rows(const uint16_t* a, int rows, int k, uint8_t* codes,
                                 float* scales, cudaStream_t s);

// y = bf16(partial[0] + partial[1]) over batch x 7168 fp32 partials (out_proj.cu).
cudaError_t launch_oproj_finish(const float* part, uint16_t* y, int batch, cudaStream_t s);


struct AttnArgs {
  const uint16_t* q;        // [batch, 64, 256] bf16
  const KvSeq* kv;          // device table
  int kv_dtype;
  float k_scale, v_scale;   // FP8 only
  const int32_t* seq_lens;  // device [batch]
  float scale;              // softmax scale
  uint16_t* out;            // [batch, 64, 256] bf16
  int batch;
  float* partials;          // slots
  int2* seq_info;           // [batch]: (first slot, splits), written for the combine kernel
  int32_t* plan;            // the split plan, written by the finish kernel's plan block
  int plan_early;           // 1: the plan was written two or more kernels earlier on the
                            // stream, so it may be read before griddepcontrol.wait
  uint32_t* err;
  int grid;
  int page_size;            // the caller's mfa_kv_cache.page_size: picks the kernel
};
// Tensor-core attention (bf16 or FP8 KV); q_map covers q as [batch * 64 rows, 256] bf16,
// boxes of [64 x 64] with 128-byte swizzle.
cudaError_t launch_attention_tc(const CUtensorMap& q_map, const AttnArgs& a, cudaStream_t s);
size_t attention_tc_smem_bytes();
// Merge of the split-K partials of every split sequence (and zero output of rejected ones);
// launched right after launch_attention_tc on the same stream, as its programmatic
// dependent.
cudaError_t launch_attention_combine(const AttnArgs& a, cudaStream_t s);

// One CTA whose bounded wait on a barrier that nothing completes gives up after limit_us
// and sets kErrTimeout in *err (selftest.cu).
cudaError_t launch_wait_selftest(uint32_t* err, uint32_t limit_us, cudaStream_t s);

// The status a set of device error bits reports (the most specific bit wins).
inline mfa_status status_of_error_bits(uint32_t bits) {
  if (bits == 0) return MFA_OK;
  if (bits & kErrCapacity) return MFA_ERR_CAPACITY;
  if (bits & kErrEmpty) return MFA_ERR_EMPTY;
  if (bits & kErrLayout) return MFA_ERR_INVALID_ARG;
  return MFA_ERR_TIMEOUT;
}

// A projection weight: bf16 stored [in, out] (scales null), or block-FP8 e4m3 codes stored
// [out, in] with one float32 scale per 128 x 128 block ([out / 128, in / 128]).
struct WRef {
  const void* ptr;
  const float* scales;
};

// The query path (x-projection onto W_qdown, finish with RMSNorm, q_up) on `s`, using the
// x-projection partials, c_hat and error word at the offsets of L inside `ws`.
mfa_status run_query_proj(const void* x, WRef w_qdown, const void* gamma, WRef w_qup, float eps,
                          void* q_out, int batch, void* ws, const WsLayout& L, cudaStream_t s);

// cuTensorMapEncodeTiled through the runtime's driver entry point (null if unavailable).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();
// 2-D bf16/uint8 tensor map over a row-major [rows, cols] matrix, box [box_cols, box_rows],
// 128-byte swizzle. Returns false if the driver rejects it. Maps already encoded on this
// host thread (same address, shape and box) are copied from a small per-thread cache.
bool encode_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, int elem_bytes,
               uint32_t box_cols, uint32_t box_rows);
// Raise `kernel`'s dynamic shared memory limit to `bytes` (the most any launch of it asks
// for) on the current device, once per device; `done` is the kernel's per-device record.
bool set_smem_limit_once(const void* kernel, int bytes, std::atomic<uint64_t>* done);
// 3-D map over a page pool [pages, page_rows, 256] (elem_bytes each), box
// [128 bytes of a row x box_rows x 1 page], 128-byte swizzle.
bool encode_pool(CUtensorMap* m, const void* base, uint64_t pages, uint64_t page_rows,
                 int elem_bytes, uint32_t box_rows);

}  // namespace mfa
