// extern "C" entry points of libmfa: argument checks, the device KV table, the workspace,
// and the kernel sequence of each call. Declarations and the contract are in include/mfa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <new>
#include <vector>

#include "mfa_internal.cuh"

// A captured decode step (include/mfa.h): the instantiated graph and the device it was
// captured on.
struct mfa_step_graph {
  cudaGraphExec_t exec;
  int device;
};

namespace mfa {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) {
    *sms = cached[dev];
    return true;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return false;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  *sms = n;
  return true;
}

// Tensor map over one sequence's cache rows: [rows, 256] elements, boxes of
// (128 bytes of a row) x kTile rows, 128-byte swizzle -- the canonical K-major /
// MN-major shared-memory layout of the tensor-core operands.
bool encode_rows(CUtensorMap* m, void* base, int rows, int dtype) {
  const int elem = dtype == MFA_KV_FP8_E4M3 ? 1 : 2;
  return encode_2d(m, base, (uint64_t)rows, kHeadDim, elem, 128 / elem, kTile);
}

mfa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MFA_OK : MFA_ERR_CUDA; }

bool valid_w8(const mfa_w8& w) {
  return w.codes != nullptr && aligned16(w.codes) && w.scales != nullptr &&
         (reinterpret_cast<uintptr_t>(w.scales) & 3u) == 0;
}

mfa_status check_kv(const mfa_kv_cache* kv) {
  if (kv == nullptr || kv->table == nullptr) return MFA_ERR_INVALID_ARG;
  if (kv->batch < 1 || kv->batch > kMaxBatch) return MFA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(kv->table) & 127u) != 0) return MFA_ERR_INVALID_ARG;
  if (kv->dtype != MFA_KV_BF16 && kv->dtype != MFA_KV_FP8_E4M3) return MFA_ERR_UNSUPPORTED;
  if (kv->dtype == MFA_KV_FP8_E4M3 && !(kv->k_scale > 0.f && kv->v_scale > 0.f))
    return MFA_ERR_INVALID_ARG;
  const int ps = kv->page_size;
  if (ps != 0 && (ps < 64 || (ps & (ps - 1)) != 0)) return MFA_ERR_INVALID_ARG;
  return MFA_OK;
}

mfa_status check_ws(void* ws, size_t ws_bytes, int batch, WsLayout* L) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MFA_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_sms(&sms)) return MFA_ERR_CUDA;
  *L = ws_layout(batch, sms);
  if (ws_bytes < L->total) return MFA_ERR_WORKSPACE;
  return MFA_OK;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// The tensor map of a weight of in_dim x out_dim: bf16 stored [in, out] (boxes [128 k x 64
// features]), or block-FP8 codes stored [out, in] (boxes [128 features x 128 k]).
bool encode_weight(CUtensorMap* m, WRef w, int in_dim, int out_dim) {
  if (w.scales != nullptr) return encode_2d(m, w.ptr, out_dim, in_dim, 1, 128, 128);
  return encode_2d(m, w.ptr, in_dim, out_dim, 2, 64, 128);
}

void set_weight_scales(WGemmArgs& p, int i, WRef w, int in_dim) {
  p.wscale[i] = w.scales;
  p.wscale_ld[i] = in_dim / 128;
}

// Where the FP8 path keeps an activation's e4m3 codes and scales (codes null: bf16 path).
struct Act8 {
  uint8_t* codes;
  float* scales;
};

// X of a projection: bf16 [batch, k] as it is, or (FP8 path) quantized into `a8` first by a
// kernel of its own; the GEMM's tensor map and scale arguments for it.
bool prepare_x(CUtensorMap* xm, WGemmArgs& p, const void* x, int batch, int k, Act8 a8,
               bool quantize, cudaStream_t s) {
  if (a8.codes == nullptr)
    return encode_2d(xm, x, (uint64_t)batch, k, 2, 64, wgemm_n_box(batch));
  if (quantize && launch_quantize_rows(static_cast<const uint16_t*>(x), batch, k, a8.codes,
                                       a8.scales, s) != cudaSuccess)
    return false;
  p.xscale = a8.scales;
  p.xscale_ld = k / 128;
  return encode_2d(xm, a8.codes, (uint64_t)batch, k, 1, 128, wgemm_n_box_fp8(batch));
}

// x [batch, 7168] onto the 128-column tiles [tile_begin, tile_end) of [W_qdown | W_k | W_v]
// (16 + 2 + 2 tiles), split-K partials into the workspace. Null weights are not read; the
// three are all bf16 (a8.codes null) or all block-FP8 (x then quantized into a8).
mfa_status run_xproj(const void* x, WRef w_qdown, WRef w_k, WRef w_v, int batch,
                     int tile_begin, int tile_end, float* part, uint32_t* err, Act8 a8,
                     cudaStream_t s) {
  CUtensorMap wm[3];
  std::memset(wm, 0, sizeof(wm));
  if (w_qdown.ptr && !encode_weight(&wm[0], w_qdown, kHidden, kRank)) return MFA_ERR_CUDA;
  if (w_k.ptr && !encode_weight(&wm[1], w_k, kHidden, kHeadDim)) return MFA_ERR_CUDA;
  if (w_v.ptr && !encode_weight(&wm[2], w_v, kHidden, kHeadDim)) return MFA_ERR_CUDA;
  WGemmArgs p{};
  CUtensorMap xm;
  if (!prepare_x(&xm, p, x, batch, kHidden, a8, true, s)) return MFA_ERR_CUDA;
  p.batch = batch;
  p.tile_begin = tile_begin;
  p.three_weights = 1;
  p.w0_tiles = kRank / 128;
  p.w1_tiles = kHeadDim / 128;
  p.kblocks_per_cta = kXProjKPerSplit / 128;
  p.out_f32 = part;
  p.out_ld = kXProjCols;
  p.err = err;
  if (w_qdown.scales != nullptr) {
    set_weight_scales(p, 0, w_qdown, kHidden);
    set_weight_scales(p, 1, w_k, kHidden);
    set_weight_scales(p, 2, w_v, kHidden);
  }
  return cuda_status(launch_wgemm(wm, xm, p, tile_end - tile_begin, kXProjSplits, s));
}

// q = bf16(c_hat W_qup): c_hat [batch, 2048], W_qup [2048, 16384], q [batch, 16384].
mfa_status run_q_up(const uint16_t* c_hat, WRef w_qup, void* q, int batch, uint32_t* err,
                    Act8 a8, cudaStream_t s) {
  CUtensorMap wm[3];
  std::memset(wm, 0, sizeof(wm));
  if (!encode_weight(&wm[0], w_qup, kRank, kQWidth)) return MFA_ERR_CUDA;
  WGemmArgs p{};
  CUtensorMap xm;
  // (the finish kernel already wrote c_hat's codes and scales on the FP8 path)
  if (!prepare_x(&xm, p, c_hat, batch, kRank, a8, false, s)) return MFA_ERR_CUDA;
  p.batch = batch;
  p.tile_begin = 0;
  p.three_weights = 0;
  p.kblocks_per_cta = kRank / 128;
  p.out_bf16 = static_cast<uint16_t*>(q);
  p.out_ld = kQWidth;
  p.err = err;
  if (w_qup.scales != nullptr) set_weight_scales(p, 0, w_qup, kRank);
  return cuda_status(launch_wgemm(wm, xm, p, kQWidth / 128, 1, s));
}


}  // namespace

mfa_status run_query_proj(const void* x, WRef w_qdown, const void* gamma, WRef w_qup, float eps,
                          void* q_out, int batch, void* ws, const WsLayout& L, cudaStream_t s) {
  float* part = at<float>(ws, L.xproj_part);
  uint32_t* err = at<uint32_t>(ws, L.err);
  const bool fp8 = w_qdown.scales != nullptr;
  const Act8 x8 = fp8 ? Act8{at<uint8_t>(ws, L.x8), at<float>(ws, L.x8_scale)} : Act8{};
  const Act8 c8 = fp8 ? Act8{at<uint8_t>(ws, L.chat8), at<float>(ws, L.chat8_scale)} : Act8{};
  mfa_status st =
      run_xproj(x, w_qdown, WRef{}, WRef{}, batch, 0, kRank / 128, part, err, x8, s);
  if (st != MFA_OK) return st;
  FinishArgs fa{};
  fa.part = part;
  fa.batch = batch;
  fa.gamma = static_cast<const uint16_t*>(gamma);
  fa.eps = eps;
  fa.c_hat = at<uint16_t>(ws, L.c_hat);
  fa.chat8 = c8.codes;
  fa.chat8_scale = c8.scales;
  fa.err = err;
  if (launch_xproj_finish(fa, s) != cudaSuccess) return MFA_ERR_CUDA;
  return run_q_up(fa.c_hat, w_qup, q_out, batch, err, c8, s);
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn != nullptr) return fn;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || p == nullptr)
    return nullptr;
  fn = reinterpret_cast<EncodeTiledFn>(p);
  return fn;
}

namespace {

// Tensor maps are pure functions of (address, shape, element size, box): each host thread
// keeps the last few it encoded, so the steady state of a serving loop (the same weights and
// buffers every step) encodes none.
struct MapKey {
  const void* base;
  uint64_t rows, cols;
  int elem_bytes;
  uint32_t box_cols, box_rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && elem_bytes == o.elem_bytes &&
           box_cols == o.box_cols && box_rows == o.box_rows;
  }
};
constexpr int kMapCache = 32;
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  int used = 0, next = 0;
};
thread_local MapCache t_maps;

}  // namespace

bool encode_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, int elem_bytes,
               uint32_t box_cols, uint32_t box_rows) {
  const MapKey key{base, rows, cols, elem_bytes, box_cols, box_rows};
  MapCache& c = t_maps;
  for (int i = 0; i < c.used; ++i) {
    if (c.key[i] == key) {
      *m = c.map[i];
      return true;
    }
  }
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(
      m, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  const int slot = c.used < kMapCache ? c.used++ : (c.next++ % kMapCache);
  c.key[slot] = key;
  c.map[slot] = *m;
  return true;
}

bool set_smem_limit_once(const void* kernel, int bytes, std::atomic<uint64_t>* done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0;
  if (bit != 0 && (done->load(std::memory_order_acquire) & bit)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  if (bit != 0) done->fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

bool encode_pool(CUtensorMap* m, const void* base, uint64_t pages, uint64_t page_rows,
                 int elem_bytes, uint32_t box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const uint64_t row_bytes = (uint64_t)kHeadDim * elem_bytes;
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)page_rows, (cuuint64_t)pages};
  cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)(row_bytes * page_rows)};
  cuuint32_t box[3] = {(cuuint32_t)(128 / elem_bytes), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(
      m, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

// The attention of one call: the tensor-core kernel, then the merge of split sequences.
// Unless the plan was launched earlier (aa.plan_early), the attention CTAs build it on chip.
mfa_status run_attention(const AttnArgs& aa, cudaStream_t s) {
  CUtensorMap q_map;
  if (!encode_2d(&q_map, aa.q, (uint64_t)aa.batch * kHeads, kHeadDim, 2, 64, 64))
    return MFA_ERR_CUDA;
  if (launch_attention_tc(q_map, aa, s) != cudaSuccess) return MFA_ERR_CUDA;
  return cuda_status(launch_attention_combine(aa, s));
}

}  // namespace
}  // namespace mfa

using namespace mfa;

extern "C" {

int32_t mfa_version(void) { return 100; }

const char* mfa_status_str(int32_t status) {
  switch (status) {
    case MFA_OK: return "MFA_OK";
    case MFA_ERR_INVALID_ARG: return "MFA_ERR_INVALID_ARG";
    case MFA_ERR_UNSUPPORTED: return "MFA_ERR_UNSUPPORTED";
    case MFA_ERR_CAPACITY: return "MFA_ERR_CAPACITY";
    case MFA_ERR_WORKSPACE: return "MFA_ERR_WORKSPACE";
    case MFA_ERR_CUDA: return "MFA_ERR_CUDA";
    case MFA_ERR_EMPTY: return "MFA_ERR_EMPTY";
    case MFA_ERR_TIMEOUT: return "MFA_ERR_TIMEOUT";
    default: return "MFA_ERR_UNKNOWN";
  }
}

size_t mfa_kv_table_bytes(int32_t batch) {
  if (batch < 1 || batch > kMaxBatch) return 0;
  return sizeof(KvSeq) * (size_t)batch;
}

mfa_status mfa_kv_table_init(void* table, size_t table_bytes, int32_t batch, int32_t dtype,
                             void* const* k_ptrs, void* const* v_ptrs,
                             const int32_t* capacity, void* stream) {
  if (batch < 1 || batch > kMaxBatch) return MFA_ERR_INVALID_ARG;
  if (table == nullptr || k_ptrs == nullptr || v_ptrs == nullptr || capacity == nullptr)
    return MFA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(table) & 127u) != 0) return MFA_ERR_INVALID_ARG;
  if (dtype != MFA_KV_BF16 && dtype != MFA_KV_FP8_E4M3) return MFA_ERR_UNSUPPORTED;
  if (table_bytes < mfa_kv_table_bytes(batch)) return MFA_ERR_WORKSPACE;
  for (int b = 0; b < batch; ++b) {
    if (k_ptrs[b] == nullptr || v_ptrs[b] == nullptr) return MFA_ERR_INVALID_ARG;
    if (!aligned16(k_ptrs[b]) || !aligned16(v_ptrs[b])) return MFA_ERR_INVALID_ARG;
    if (capacity[b] < 1 || capacity[b] > MFA_MAX_CONTEXT) return MFA_ERR_INVALID_ARG;
  }
  if (encode_tiled_fn() == nullptr) return MFA_ERR_CUDA;
  std::vector<KvSeq> host(batch);
  std::memset(host.data(), 0, sizeof(KvSeq) * batch);
  for (int b = 0; b < batch; ++b) {
    if (!encode_rows(&host[b].tmap_k, k_ptrs[b], capacity[b], dtype) ||
        !encode_rows(&host[b].tmap_v, v_ptrs[b], capacity[b], dtype))
      return MFA_ERR_INVALID_ARG;
    host[b].k = k_ptrs[b];
    host[b].v = v_ptrs[b];
    host[b].capacity = capacity[b];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(table, host.data(), sizeof(KvSeq) * batch,
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

mfa_status mfa_kv_table_init_paged(void* table, size_t table_bytes, int32_t batch,
                                   int32_t dtype, void* k_pool, void* v_pool, int32_t num_pages,
                                   int32_t page_size, const int32_t* page_table,
                                   int32_t max_pages, const int32_t* pages_per_seq,
                                   void* stream) {
  if (batch < 1 || batch > kMaxBatch) return MFA_ERR_INVALID_ARG;
  if (table == nullptr || k_pool == nullptr || v_pool == nullptr || page_table == nullptr ||
      pages_per_seq == nullptr)
    return MFA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(table) & 127u) != 0) return MFA_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) != 0)
    return MFA_ERR_INVALID_ARG;
  if (dtype != MFA_KV_BF16 && dtype != MFA_KV_FP8_E4M3) return MFA_ERR_UNSUPPORTED;
  if (page_size < 64 || (page_size & (page_size - 1)) != 0 || page_size > MFA_MAX_CONTEXT)
    return MFA_ERR_UNSUPPORTED;
  if (num_pages < 1 || max_pages < 1) return MFA_ERR_INVALID_ARG;
  if (table_bytes < mfa_kv_table_bytes(batch)) return MFA_ERR_WORKSPACE;
  for (int b = 0; b < batch; ++b) {
    const int64_t cap = (int64_t)pages_per_seq[b] * page_size;
    if (pages_per_seq[b] < 1 || pages_per_seq[b] > max_pages || cap > MFA_MAX_CONTEXT)
      return MFA_ERR_INVALID_ARG;
  }
  if (encode_tiled_fn() == nullptr) return MFA_ERR_CUDA;
  const int elem = dtype == MFA_KV_FP8_E4M3 ? 1 : 2;
  KvSeq proto;
  std::memset(&proto, 0, sizeof(proto));
  if (!encode_pool(&proto.tmap_k, k_pool, num_pages, page_size, elem,
                   paged_box_rows(page_size)) ||
      !encode_pool(&proto.tmap_v, v_pool, num_pages, page_size, elem,
                   paged_box_rows(page_size)))
    return MFA_ERR_INVALID_ARG;
  proto.k = k_pool;
  proto.v = v_pool;
  proto.page_size = page_size;
  proto.num_pages = num_pages;
  std::vector<KvSeq> host(batch, proto);
  for (int b = 0; b < batch; ++b) {
    host[b].capacity = pages_per_seq[b] * page_size;
    host[b].pages = page_table + (size_t)b * max_pages;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(table, host.data(), sizeof(KvSeq) * batch,
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

size_t mfa_workspace_bytes(int32_t batch) {
  if (batch < 1 || batch > kMaxBatch) return 0;
  int sms = 0;
  if (!device_sms(&sms)) return 0;
  return ws_layout(batch, sms).total;
}

mfa_status mfa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MFA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

mfa_status mfa_get_error(void* ws, void* stream) {
  if (ws == nullptr) return MFA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MFA_ERR_CUDA;
  uint32_t bits = 0;
  if (cudaMemcpy(&bits, ws, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (bits == 0) return MFA_OK;
  if (cudaMemsetAsync(ws, 0, sizeof(bits), s) != cudaSuccess) return MFA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MFA_ERR_CUDA;
  return status_of_error_bits(bits);
}

mfa_status mfa_query_proj(const void* x, const void* w_qdown, const void* gamma,
                          const void* w_qup, float eps, void* q_out, int32_t batch,
                          void* ws, size_t ws_bytes, void* stream) {
  if (batch < 1 || batch > kMaxBatch) return MFA_ERR_INVALID_ARG;
  if (!(eps > 0.f)) return MFA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_qdown, gamma, w_qup, q_out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MFA_ERR_INVALID_ARG;
  WsLayout L;
  mfa_status st = check_ws(ws, ws_bytes, batch, &L);
  if (st != MFA_OK) return st;
  return run_query_proj(x, WRef{w_qdown, nullptr}, gamma, WRef{w_qup, nullptr}, eps, q_out,
                        batch, ws, L, static_cast<cudaStream_t>(stream));
}

mfa_status mfa_query_proj_w8(const void* x, mfa_w8 w_qdown, const void* gamma, mfa_w8 w_qup,
                             float eps, void* q_out, int32_t batch, void* ws, size_t ws_bytes,
                             void* stream) {
  if (batch < 1 || batch > kMaxBatch) return MFA_ERR_INVALID_ARG;
  if (!(eps > 0.f)) return MFA_ERR_INVALID_ARG;
  const void* ptrs[] = {x, gamma, q_out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MFA_ERR_INVALID_ARG;
  if (!valid_w8(w_qdown) || !valid_w8(w_qup)) return MFA_ERR_INVALID_ARG;
  WsLayout L;
  mfa_status st = check_ws(ws, ws_bytes, batch, &L);
  if (st != MFA_OK) return st;
  return run_query_proj(x, WRef{w_qdown.codes, w_qdown.scales}, gamma,
                        WRef{w_qup.codes, w_qup.scales}, eps, q_out, batch, ws, L,
                        static_cast<cudaStream_t>(stream));
}

mfa_status mfa_kv_append(const void* x, const void* w_k, const void* w_v,
                         const mfa_kv_cache* kv, const int32_t* pos, void* ws,
                         size_t ws_bytes, void* stream) {
  mfa_status st = check_kv(kv);
  if (st != MFA_OK) return st;
  const void* ptrs[] = {x, w_k, w_v, pos};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MFA_ERR_INVALID_ARG;
  WsLayout L;
  st = check_ws(ws, ws_bytes, kv->batch, &L);
  if (st != MFA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = at<float>(ws, L.xproj_part);
  st = run_xproj(x, WRef{}, WRef{w_k, nullptr}, WRef{w_v, nullptr}, kv->batch, kRank / 128,
                 kXProjCols / 128, part, at<uint32_t>(ws, L.err), Act8{}, s);
  if (st != MFA_OK) return st;
  FinishArgs fa{};
  fa.part = part;
  fa.batch = kv->batch;
  fa.kv = static_cast<const KvSeq*>(kv->table);
  fa.kv_dtype = kv->dtype;
  fa.k_scale = kv->k_scale;
  fa.v_scale = kv->v_scale;
  fa.pos = pos;
  fa.pos_from_len = 0;
  fa.err = at<uint32_t>(ws, L.err);
  return cuda_status(launch_xproj_finish(fa, s));
}

mfa_status mfa_decode_attn(const void* q, const mfa_kv_cache* kv, const int32_t* seq_lens,
                           float scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  mfa_status st = check_kv(kv);
  if (st != MFA_OK) return st;
  if (!(scale > 0.f)) return MFA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, seq_lens, out};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MFA_ERR_INVALID_ARG;
  WsLayout L;
  st = check_ws(ws, ws_bytes, kv->batch, &L);
  if (st != MFA_OK) return st;
  AttnArgs aa{};
  aa.q = static_cast<const uint16_t*>(q);
  aa.kv = static_cast<const KvSeq*>(kv->table);
  aa.kv_dtype = kv->dtype;
  aa.k_scale = kv->k_scale;
  aa.v_scale = kv->v_scale;
  aa.seq_lens = seq_lens;
  aa.scale = scale;
  aa.out = static_cast<uint16_t*>(out);
  aa.batch = kv->batch;
  aa.partials = at<float>(ws, L.attn_part);
  aa.seq_info = at<int2>(ws, L.seq_info);
  aa.plan = at<int32_t>(ws, L.plan);
  aa.plan_early = 0;
  aa.err = at<uint32_t>(ws, L.err);
  aa.grid = L.attn_grid;
  aa.page_size = kv->page_size;
  return run_attention(aa, static_cast<cudaStream_t>(stream));
}

mfa_status mfa_o_proj(const void* out, const void* w_o, void* y, int32_t batch, void* ws,
                      size_t ws_bytes, void* stream) {
  if (batch < 1 || batch > kMaxBatch) return MFA_ERR_INVALID_ARG;
  const void* ptrs[] = {out, w_o, y};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MFA_ERR_INVALID_ARG;
  WsLayout L;
  mfa_status st = check_ws(ws, ws_bytes, batch, &L);
  if (st != MFA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // W_o^T tiles of 128 output features on the M side, out [batch, 16384] on the N side
  CUtensorMap wm[3];
  std::memset(wm, 0, sizeof(wm));
  if (!encode_2d(&wm[0], w_o, kQWidth, kHidden, 2, 64, 128)) return MFA_ERR_CUDA;
  CUtensorMap xm;
  if (!encode_2d(&xm, out, (uint64_t)batch, kQWidth, 2, 64, wgemm_n_box(batch)))
    return MFA_ERR_CUDA;
  float* part = at<float>(ws, L.oproj_part);
  WGemmArgs p{};
  p.batch = batch;
  p.tile_begin = 0;
  p.three_weights = 0;
  p.kblocks_per_cta = kOProjKPerSplit / 128;
  p.out_f32 = part;
  p.out_ld = kHidden;
  p.err = at<uint32_t>(ws, L.err);
  if (launch_wgemm(wm, xm, p, kHidden / 128, kOProjSplits, s) != cudaSuccess)
    return MFA_ERR_CUDA;
  return cuda_status(launch_oproj_finish(part, static_cast<uint16_t*>(y), batch, s));
}

}  // extern "C"

namespace mfa {
namespace {

// The whole decode step after the host-side checks: x-projection, finish (RMSNorm, append,
// split plan), q_up, attention, combine.
mfa_status decode_layer_impl(const void* x, WRef w_qdown, const void* gamma, WRef w_qup,
                             WRef w_k, WRef w_v, float eps, const mfa_kv_cache* kv,
                             const int32_t* seq_lens, float scale, void* q_out, void* out,
                             void* ws, const WsLayout& L, cudaStream_t s) {
  mfa_status st;
  const int batch = kv->batch;
  AttnArgs aa{};
  aa.q = static_cast<const uint16_t*>(q_out);
  aa.kv = static_cast<const KvSeq*>(kv->table);
  aa.kv_dtype = kv->dtype;
  aa.k_scale = kv->k_scale;
  aa.v_scale = kv->v_scale;
  aa.seq_lens = seq_lens;
  aa.scale = scale;
  aa.out = static_cast<uint16_t*>(out);
  aa.batch = batch;
  aa.partials = at<float>(ws, L.attn_part);
  aa.seq_info = at<int2>(ws, L.seq_info);
  aa.plan = at<int32_t>(ws, L.plan);
  aa.plan_early = 1;
  aa.err = at<uint32_t>(ws, L.err);
  aa.grid = L.attn_grid;
  aa.page_size = kv->page_size;
  // one projection of x onto [W_qdown | W_k | W_v]
  float* part = at<float>(ws, L.xproj_part);
  const bool fp8 = w_qdown.scales != nullptr;
  const Act8 x8 = fp8 ? Act8{at<uint8_t>(ws, L.x8), at<float>(ws, L.x8_scale)} : Act8{};
  const Act8 c8 = fp8 ? Act8{at<uint8_t>(ws, L.chat8), at<float>(ws, L.chat8_scale)} : Act8{};
  st = run_xproj(x, w_qdown, w_k, w_v, batch, 0, kXProjCols / 128, part,
                 at<uint32_t>(ws, L.err), x8, s);
  if (st != MFA_OK) return st;
  // split-K sums, RMSNorm of the query half, K/V append at row seq_lens[b] - 1
  FinishArgs fa{};
  fa.part = part;
  fa.batch = batch;
  fa.gamma = static_cast<const uint16_t*>(gamma);
  fa.eps = eps;
  fa.c_hat = at<uint16_t>(ws, L.c_hat);
  fa.chat8 = c8.codes;
  fa.chat8_scale = c8.scales;
  fa.kv = static_cast<const KvSeq*>(kv->table);
  fa.kv_dtype = kv->dtype;
  fa.k_scale = kv->k_scale;
  fa.v_scale = kv->v_scale;
  fa.pos = seq_lens;
  fa.pos_from_len = 1;
  fa.err = at<uint32_t>(ws, L.err);
  // plus the attention's split plan (it needs only seq_lens and the KV table), which the
  // attention kernel two launches later reads before waiting on its predecessor
  fa.plan = aa.plan;
  fa.seq_info = aa.seq_info;
  fa.attn_grid = aa.grid;
  if (launch_xproj_finish(fa, s) != cudaSuccess) return MFA_ERR_CUDA;
  st = run_q_up(fa.c_hat, w_qup, q_out, batch, fa.err, c8, s);
  if (st != MFA_OK) return st;
  return run_attention(aa, s);
}

}  // namespace
}  // namespace mfa

namespace mfa {
namespace {

// The checks of one decode step (direct or captured), in this order: the KV description, eps
// and scale, the pointers (non-null, 16-byte aligned), the FP8 weights (weights_ok), then the
// workspace, whose layout goes to *L.
mfa_status check_layer(const void* const* ptrs, size_t n, bool weights_ok, float eps,
                       float scale, const mfa_kv_cache* kv, void* ws, size_t ws_bytes,
                       WsLayout* L) {
  mfa_status st = check_kv(kv);
  if (st != MFA_OK) return st;
  if (!(eps > 0.f) || !(scale > 0.f)) return MFA_ERR_INVALID_ARG;
  for (size_t i = 0; i < n; ++i)
    if (ptrs[i] == nullptr || !aligned16(ptrs[i])) return MFA_ERR_INVALID_ARG;
  if (!weights_ok) return MFA_ERR_INVALID_ARG;
  return check_ws(ws, ws_bytes, kv->batch, L);
}

bool valid_w8_all(const mfa_w8& a, const mfa_w8& b, const mfa_w8& c, const mfa_w8& d) {
  return valid_w8(a) && valid_w8(b) && valid_w8(c) && valid_w8(d);
}

// Records launch(stream) on a stream of the library's own (thread-local capture, so other
// threads' work is not affected) and instantiates the graph for the current device.
template <class F>
mfa_status capture_step(F&& launch, mfa_step_graph** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MFA_ERR_CUDA;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return MFA_ERR_CUDA;
  mfa_status st = MFA_ERR_CUDA;
  cudaGraph_t graph = nullptr;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) == cudaSuccess) {
    st = launch(cs);
    // the capture always ends, whatever the launches returned
    if (cudaStreamEndCapture(cs, &graph) != cudaSuccess && st == MFA_OK) st = MFA_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  if (st == MFA_OK && (graph == nullptr || cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess))
    st = MFA_ERR_CUDA;
  if (graph != nullptr) cudaGraphDestroy(graph);
  cudaStreamDestroy(cs);
  if (st != MFA_OK) return st;
  mfa_step_graph* g = new (std::nothrow) mfa_step_graph{exec, dev};
  if (g == nullptr) {
    cudaGraphExecDestroy(exec);
    return MFA_ERR_CUDA;
  }
  *out = g;
  return MFA_OK;
}

}  // namespace
}  // namespace mfa

extern "C" {

mfa_status mfa_decode_layer(const void* x, const void* w_qdown, const void* gamma,
                            const void* w_qup, const void* w_k, const void* w_v, float eps,
                            const mfa_kv_cache* kv, const int32_t* seq_lens, float scale,
                            void* q_out, void* out, void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {x, w_qdown, gamma, w_qup, w_k, w_v, seq_lens, q_out, out};
  WsLayout L;
  const mfa_status st = check_layer(ptrs, 9, true, eps, scale, kv, ws, ws_bytes, &L);
  if (st != MFA_OK) return st;
  return decode_layer_impl(x, WRef{w_qdown, nullptr}, gamma, WRef{w_qup, nullptr},
                           WRef{w_k, nullptr}, WRef{w_v, nullptr}, eps, kv, seq_lens, scale,
                           q_out, out, ws, L, static_cast<cudaStream_t>(stream));
}

mfa_status mfa_decode_layer_w8(const void* x, mfa_w8 w_qdown, const void* gamma, mfa_w8 w_qup,
                               mfa_w8 w_k, mfa_w8 w_v, float eps, const mfa_kv_cache* kv,
                               const int32_t* seq_lens, float scale, void* q_out, void* out,
                               void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {x, gamma, seq_lens, q_out, out};
  WsLayout L;
  const bool w_ok = valid_w8_all(w_qdown, w_qup, w_k, w_v);
  const mfa_status st = check_layer(ptrs, 5, w_ok, eps, scale, kv, ws, ws_bytes, &L);
  if (st != MFA_OK) return st;
  return decode_layer_impl(x, WRef{w_qdown.codes, w_qdown.scales}, gamma,
                           WRef{w_qup.codes, w_qup.scales}, WRef{w_k.codes, w_k.scales},
                           WRef{w_v.codes, w_v.scales}, eps, kv, seq_lens, scale, q_out, out,
                           ws, L, static_cast<cudaStream_t>(stream));
}

mfa_status mfa_decode_layer_graph(const void* x, const void* w_qdown, const void* gamma,
                                  const void* w_qup, const void* w_k, const void* w_v, float eps,
                                  const mfa_kv_cache* kv, const int32_t* seq_lens, float scale,
                                  void* q_out, void* out, void* ws, size_t ws_bytes,
                                  mfa_step_graph** graph) {
  if (graph == nullptr) return MFA_ERR_INVALID_ARG;
  *graph = nullptr;
  const void* ptrs[] = {x, w_qdown, gamma, w_qup, w_k, w_v, seq_lens, q_out, out};
  WsLayout L;
  const mfa_status st = check_layer(ptrs, 9, true, eps, scale, kv, ws, ws_bytes, &L);
  if (st != MFA_OK) return st;
  return capture_step(
      [&](cudaStream_t cs) {
        return decode_layer_impl(x, WRef{w_qdown, nullptr}, gamma, WRef{w_qup, nullptr},
                                 WRef{w_k, nullptr}, WRef{w_v, nullptr}, eps, kv, seq_lens,
                                 scale, q_out, out, ws, L, cs);
      },
      graph);
}

mfa_status mfa_decode_layer_w8_graph(const void* x, mfa_w8 w_qdown, const void* gamma,
                                     mfa_w8 w_qup, mfa_w8 w_k, mfa_w8 w_v, float eps,
                                     const mfa_kv_cache* kv, const int32_t* seq_lens,
                                     float scale, void* q_out, void* out, void* ws,
                                     size_t ws_bytes, mfa_step_graph** graph) {
  if (graph == nullptr) return MFA_ERR_INVALID_ARG;
  *graph = nullptr;
  const void* ptrs[] = {x, gamma, seq_lens, q_out, out};
  WsLayout L;
  const bool w_ok = valid_w8_all(w_qdown, w_qup, w_k, w_v);
  const mfa_status st = check_layer(ptrs, 5, w_ok, eps, scale, kv, ws, ws_bytes, &L);
  if (st != MFA_OK) return st;
  return capture_step(
      [&](cudaStream_t cs) {
        return decode_layer_impl(x, WRef{w_qdown.codes, w_qdown.scales}, gamma,
                                 WRef{w_qup.codes, w_qup.scales}, WRef{w_k.codes, w_k.scales},
                                 WRef{w_v.codes, w_v.scales}, eps, kv, seq_lens, scale, q_out,
                                 out, ws, L, cs);
      },
      graph);
}

mfa_status mfa_step_graph_launch(const mfa_step_graph* graph, void* stream) {
  if (graph == nullptr) return MFA_ERR_INVALID_ARG;
  return cuda_status(cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)));
}

void mfa_step_graph_destroy(mfa_step_graph* graph) {
  if (graph == nullptr) return;
  cudaGraphExecDestroy(graph->exec);
  delete graph;
}

}  // extern "C"
