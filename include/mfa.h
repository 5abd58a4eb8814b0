/*
 * mfa.h -- C ABI of the B200 (sm_100a) decode step of Step-3's MFA attention layer.
 *
 * The layer (Step-3 pages: bud-325 summary, "Key claims" and "Method"; redeep.blog,
 * "What's New" and the architecture table): for each token, the hidden vector x (7168) is
 * projected down to a low-rank query of width 2048, normalized, and projected up to 64
 * query heads of dimension 256. All 64 heads attend over ONE shared K head and ONE shared
 * V head (dimension 256) kept in a per-sequence KV cache, which holds one K and one V
 * vector per token; the new token's K and V are projected from x and appended.
 *
 * Readings taken where the pages are silent (stated once here, used by every call):
 *   - "normalized" = RMSNorm over the 2048 values: c_hat = c / sqrt(mean(c^2) + eps) * gamma;
 *   - k = x W_k, v = x W_v with W_k, W_v of shape [7168, 256]; no positional encoding;
 *   - softmax scale is an argument (1/sqrt(256) = 1/16 for the layer);
 *   - weights are row-major [in, out]; head h of q is columns [256 h, 256 h + 256);
 *   - seq_lens[b] counts the positions attended AFTER the append; the new token is
 *     written at row seq_lens[b] - 1 and attended to;
 *   - FP8 caches store e4m3(value / scale), one float scale per tensor for K and for V;
 *   - every rounding (fp32 -> bf16, fp32 -> e4m3) is to nearest, ties to even; e4m3
 *     saturates to +-448.
 *
 * Conventions for every call:
 *   - "device" pointers are CUDA global-memory addresses on the current device; "host"
 *     pointers are ordinary CPU memory. All buffers are owned by the caller; the library
 *     keeps no pointer after a call returns.
 *   - bf16 buffers hold raw bfloat16 bit patterns (uint16_t). Every device buffer must
 *     be 16-byte aligned; rows are dense (no padding) unless stated.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Compute calls only
 *     enqueue work on it: they neither allocate nor synchronize, and may be captured in
 *     a CUDA graph. Setup calls (mfa_kv_table_init, mfa_workspace_init, and the capture
 *     calls mfa_decode_layer_graph / _w8_graph, which create a stream and a CUDA graph of
 *     their own) may synchronize.
 *   - Problems visible on the host (null pointer, bad size, misalignment, workspace too
 *     small, unsupported dtype) return an error status before anything is enqueued.
 *     Problems visible only on the device (a length above a sequence's capacity, an empty
 *     sequence, a bounded wait that expired) set a flag in the workspace and the affected
 *     sequences' outputs are zero-filled; mfa_get_error reports and clears it.
 *   - No call aborts, throws or prints.
 */
#ifndef MFA_H_
#define MFA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MFA_API __attribute__((visibility("default")))
#else
#define MFA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Layer dimensions stated on the pages (bud-325 "Key claims"; redeep architecture table). */
#define MFA_HIDDEN 7168      /* hidden width of x */
#define MFA_Q_RANK 2048      /* low-rank query width */
#define MFA_N_HEADS 64       /* query heads */
#define MFA_HEAD_DIM 256     /* dimension of every query head and of the shared K and V head */
#define MFA_MAX_CONTEXT 65536 /* longest context the model takes (redeep architecture table) */
/* Library limit: sequences per call (the attention kernel plans the batch on chip). */
#define MFA_MAX_BATCH 1024

typedef enum {
  MFA_OK = 0,
  MFA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, size out of range, eps <= 0, ... */
  MFA_ERR_UNSUPPORTED = 2, /* unknown KV dtype, or no sm_100 device */
  MFA_ERR_CAPACITY = 3,    /* device: a length/position outside a sequence's capacity */
  MFA_ERR_WORKSPACE = 4,   /* workspace or table buffer too small */
  MFA_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed (launch error, ...) */
  MFA_ERR_EMPTY = 6,       /* device: a sequence with seq_lens[b] == 0 in mfa_decode_attn */
  MFA_ERR_TIMEOUT = 7      /* device: a bounded wait inside a kernel expired */
} mfa_status;

typedef enum {
  MFA_KV_BF16 = 0,     /* cache rows are 256 bfloat16 values (512 bytes) */
  MFA_KV_FP8_E4M3 = 1  /* cache rows are 256 OCP e4m3 codes (256 bytes) */
} mfa_kv_dtype;

/* Description of a KV cache of `batch` sequences, passed by pointer to the compute calls.
 * `table` is the device table written by mfa_kv_table_init for the same batch and dtype. */
typedef struct {
  int32_t batch;
  int32_t dtype;       /* mfa_kv_dtype */
  float k_scale;       /* FP8 only: K rows hold e4m3(k / k_scale); must be > 0 */
  float v_scale;       /* FP8 only: V rows hold e4m3(v / v_scale); must be > 0 */
  const void* table;   /* device */
  int32_t page_size;   /* 0 for a table of mfa_kv_table_init, the page size for one of
                          mfa_kv_table_init_paged (it picks the kernel; a value the table
                          contradicts computes no attention and sets MFA_ERR_INVALID_ARG in
                          the workspace) */
} mfa_kv_cache;

/* ---------------------------------------------------------------------------------------
 * Setup
 * ------------------------------------------------------------------------------------- */

/* Library version (major * 10000 + minor * 100 + patch). */
MFA_API int32_t mfa_version(void);

/* Human-readable name of a status code (static string, never NULL). */
MFA_API const char* mfa_status_str(int32_t status);

/* Bytes of the device KV table for `batch` sequences (0 if batch is out of range). */
MFA_API size_t mfa_kv_table_bytes(int32_t batch);

/* Describe a KV cache to the library. For each sequence b: k_ptrs[b] and v_ptrs[b] are
 * device base addresses of its K and V rows, each [capacity[b], 256] elements of `dtype`,
 * row-major, 16-byte aligned (sequences may live in separate allocations or be slices of
 * one [B, L, 256] buffer). k_ptrs, v_ptrs and capacity are HOST arrays of length `batch`;
 * 1 <= capacity[b] <= MFA_MAX_CONTEXT.
 * `table` is a DEVICE buffer of at least mfa_kv_table_bytes(batch) bytes, 128-byte
 * aligned. The call encodes one TMA tensor map per K and V buffer on the host, copies the
 * table to `table` on `stream` and waits for that copy. Call it again whenever a
 * sequence's buffer moves or grows. Errors: INVALID_ARG, WORKSPACE (table too small),
 * UNSUPPORTED (dtype), CUDA (no device / driver entry point / copy failure). */
MFA_API mfa_status mfa_kv_table_init(void* table, size_t table_bytes, int32_t batch, int32_t dtype,
                             void* const* k_ptrs, void* const* v_ptrs,
                             const int32_t* capacity, void* stream);

/* Describe a paged KV cache, the block-table layout of serving engines (step3-fp8 model
 * page, "Deployment": inference with vLLM and SGLang, which both keep the KV cache in
 * fixed-size pages listed per sequence in a page table). k_pool and v_pool
 * are DEVICE buffers [num_pages, page_size, 256] of `dtype`, 16-byte aligned; row j of
 * sequence b is row j % page_size of page page_table[b * max_pages + j / page_size].
 * page_table: DEVICE int32 [batch, max_pages] (4-byte aligned), read by the kernels (not
 * copied): its contents may change between calls, e.g. when a sequence gets a new page.
 * pages_per_seq: HOST int32 [batch], the pages given to each sequence (1..max_pages); the
 * sequence's capacity is pages_per_seq[b] * page_size <= MFA_MAX_CONTEXT.
 * page_size: a power of two, at least 64 (64-row pages take two TMA operations per
 * 128-position window, larger pages one).
 * Rows of a sequence's pages past its length may hold any bytes, NaN included: attention
 * never weights them, and the values it loads for them are zeroed on chip before the
 * tensor core multiplies by a zero weight. An append whose page id is outside
 * [0, num_pages) writes nothing and sets MFA_ERR_CAPACITY; the attention reads such pages
 * as zeros. `table` as in mfa_kv_table_init; the call waits for its copy. Errors:
 * INVALID_ARG, UNSUPPORTED (dtype, or page_size not a power of two >= 64), WORKSPACE
 * (table too small), CUDA. */
MFA_API mfa_status mfa_kv_table_init_paged(void* table, size_t table_bytes, int32_t batch,
                                           int32_t dtype, void* k_pool, void* v_pool,
                                           int32_t num_pages, int32_t page_size,
                                           const int32_t* page_table, int32_t max_pages,
                                           const int32_t* pages_per_seq, void* stream);

/* Bytes of the workspace the compute calls need for `batch` sequences on the current
 * device (0 if batch is out of range). One workspace must not be used by two calls that
 * can run at the same time. */
MFA_API size_t mfa_workspace_bytes(int32_t batch);

/* Zero a freshly allocated workspace (device buffer, 256-byte aligned) on `stream` and
 * wait. Needed once per allocation: the compute calls leave it ready for the next call. */
MFA_API mfa_status mfa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Wait for `stream`, then report and clear the device-side error flags of `ws`:
 * MFA_OK, MFA_ERR_CAPACITY, MFA_ERR_EMPTY, MFA_ERR_INVALID_ARG (an mfa_kv_cache whose
 * page_size the table contradicts) or MFA_ERR_TIMEOUT (the first set, in that order), or
 * MFA_ERR_CUDA if the stream reports an error. */
MFA_API mfa_status mfa_get_error(void* ws, void* stream);

/* ---------------------------------------------------------------------------------------
 * Compute (asynchronous on `stream`)
 * ------------------------------------------------------------------------------------- */

/* MFA query path (pages: bud-325 "Method" -- down-projection 7168 -> 2048, normalization,
 * up-projection to 64 heads x 256):
 *   c = x W_qdown (fp32 accumulation); c_hat = bf16(c / sqrt(mean(c^2) + eps) * gamma);
 *   q = bf16(c_hat W_qup), written as q_out[b][h][j] = q[b][256 h + j].
 * x: device bf16 [batch, 7168]; w_qdown: device bf16 [7168, 2048]; gamma: device bf16
 * [2048]; w_qup: device bf16 [2048, 16384]; q_out: device bf16 [batch, 64, 256].
 * 1 <= batch <= MFA_MAX_BATCH; eps > 0 (1e-6 for the layer).
 * ws: device workspace of mfa_workspace_bytes(batch) bytes (initialized once). */
MFA_API mfa_status mfa_query_proj(const void* x, const void* w_qdown, const void* gamma,
                          const void* w_qup, float eps, void* q_out, int32_t batch,
                          void* ws, size_t ws_bytes, void* stream);

/* Shared K/V head projection and cache append (pages: bud-325 "Method" -- one K and one
 * V per token, shared by all query heads):
 *   k = x W_k, v = x W_v (fp32 accumulation), stored as bf16(k) / bf16(v), or as
 *   e4m3(k / k_scale) / e4m3(v / v_scale), at row pos[b] of sequence b.
 * x: device bf16 [kv->batch, 7168]; w_k, w_v: device bf16 [7168, 256]; pos: device int32
 * [kv->batch]. A position outside [0, capacity[b]) writes nothing for that sequence and
 * sets MFA_ERR_CAPACITY in the workspace. Only the row pos[b] of each cache is written. */
MFA_API mfa_status mfa_kv_append(const void* x, const void* w_k, const void* w_v,
                         const mfa_kv_cache* kv, const int32_t* pos, void* ws,
                         size_t ws_bytes, void* stream);

/* Decode attention of the 64 query heads over the shared K/V head (pages: bud-325
 * "Method"; the cost is max(attention compute, KV memory access)):
 *   out[b][h] = sum_{j < L_b} softmax_j(scale * q[b][h] . K_b[j]) V_b[j],  L_b = seq_lens[b],
 * with K_b, V_b the cache rows (e4m3 codes times their scale for FP8 caches). For FP8 caches
 * the products run on e4m3 tensor cores: the cached codes are used exactly; q is written as
 * a pair of e4m3 values (hi + lo, one power-of-two scale per sequence), exact for every
 * element within 2^-10 of the sequence's largest |q|; the softmax weights as such a pair
 * within 2^-8 of their value (a bf16 rounding's size).
 * q: device bf16 [kv->batch, 64, 256]; seq_lens: device int32 [kv->batch]; out: device
 * bf16 [kv->batch, 64, 256]; scale > 0 (1/16 for the layer). The work is split over the
 * GPU's SMs by length (split-K over the cache; a second kernel on the same stream merges
 * the splits). A sequence with
 * L_b == 0 or L_b > capacity[b] gets a zero output and sets MFA_ERR_EMPTY /
 * MFA_ERR_CAPACITY in the workspace. */
MFA_API mfa_status mfa_decode_attn(const void* q, const mfa_kv_cache* kv, const int32_t* seq_lens,
                           float scale, void* out, void* ws, size_t ws_bytes, void* stream);

/* One whole MFA decode step: mfa_query_proj, then mfa_kv_append at row seq_lens[b] - 1,
 * then mfa_decode_attn over seq_lens[b] rows -- in that order, on `stream`.
 * Arguments as in those calls; q_out (device bf16 [batch, 64, 256]) receives q.
 * The library does not advance seq_lens: that is the caller's bookkeeping. */
MFA_API mfa_status mfa_decode_layer(const void* x, const void* w_qdown, const void* gamma,
                            const void* w_qup, const void* w_k, const void* w_v, float eps,
                            const mfa_kv_cache* kv, const int32_t* seq_lens, float scale,
                            void* q_out, void* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Block-FP8 weights
 * ------------------------------------------------------------------------------------- */

/* A block-FP8 projection weight (step3-fp8 model page, "Deployment": the checkpoints are
 * stored in bf16 and in block-fp8; the Step-3 pages: the whole model runs in FP8). The pages
 * give neither block size nor arithmetic; the library's reading: e4m3 codes in the
 * checkpoints' [out, in] order (row-major, out rows of `in` codes) with one float32 scale per
 * 128 x 128 block, and the projection runs in FP8: its input row is quantized per group of
 * 128 values (scale = max |a| / 448, code = e4m3(a / scale), both float32 operations rounded
 * to nearest even, the code saturating), the tensor cores multiply codes (e4m3 x e4m3, float32
 * accumulation), and each 128-wide block of the sum is scaled by its weight and activation
 * scales: y = sum over blocks of s_w s_a sum(code_w code_a). The RMSNorm, the K/V cache and the
 * attention are as in the bf16 calls. The weights stream from HBM as codes (half the bytes). */
typedef struct {
  const void* codes;    /* device uint8 [out, in], 16-byte aligned */
  const float* scales;  /* device float32 [out / 128, in / 128] (row-major), 4-byte aligned */
} mfa_w8;

/* mfa_query_proj on the FP8 path: block-FP8 W_qdown (codes [2048, 7168], scales [16, 56])
 * and W_qup (codes [16384, 2048], scales [128, 16]); x and c_hat quantized as above.
 * Errors as mfa_query_proj. */
MFA_API mfa_status mfa_query_proj_w8(const void* x, mfa_w8 w_qdown, const void* gamma,
                                     mfa_w8 w_qup, float eps, void* q_out, int32_t batch,
                                     void* ws, size_t ws_bytes, void* stream);

/* mfa_decode_layer on the FP8 path: W_qdown and W_qup as in mfa_query_proj_w8, W_k and W_v
 * codes [256, 7168] with scales [2, 56]. Errors as mfa_decode_layer. */
MFA_API mfa_status mfa_decode_layer_w8(const void* x, mfa_w8 w_qdown, const void* gamma,
                                       mfa_w8 w_qup, mfa_w8 w_k, mfa_w8 w_v, float eps,
                                       const mfa_kv_cache* kv, const int32_t* seq_lens,
                                       float scale, void* q_out, void* out, void* ws,
                                       size_t ws_bytes, void* stream);

/* Output projection of the attention (pages: bud-325 "Method" -- the per-token decoding
 * cost counts the linear projections around attention, and each layer's attention hands a
 * hidden-width vector to the FFN; the 16384 -> 7168 shape is the reading that the 64 x 256
 * head outputs return to the hidden width 7168):
 *   y = bf16(out W_o), fp32 accumulation.
 * out: device bf16 [batch, 64 * 256] (the attention output, heads in order, as written by
 * mfa_decode_attn / mfa_decode_layer); w_o: device bf16 [16384, 7168], row-major [in, out];
 * y: device bf16 [batch, 7168]. 1 <= batch <= MFA_MAX_BATCH.
 * ws: device workspace of mfa_workspace_bytes(batch) bytes (initialized once); it holds the
 * split-K partials. Errors: INVALID_ARG (null/misaligned pointer, batch out of range),
 * WORKSPACE (ws too small), CUDA (launch failure). */
MFA_API mfa_status mfa_o_proj(const void* out, const void* w_o, void* y, int32_t batch,
                              void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Without a caller-provided workspace
 * ------------------------------------------------------------------------------------- */

/* Largest batch mfa_query_proj_noalloc accepts. */
#define MFA_NOALLOC_MAX_BATCH 32

/* mfa_query_proj without the workspace, for callers that cannot allocate device memory:
 * programs whose device memory is planned once, up front, by another component (a serving
 * engine that gives all free HBM to its KV cache); loops that must not call the allocator
 * once running, because cudaMalloc can synchronize the device and take unbounded time; and
 * plugin interfaces that pass inputs and outputs but no workspace. The Step-3 pages have no
 * counterpart to this call: it is a convenience of the library, not a step of the method.
 * Arguments, results and rounding are those of mfa_query_proj without ws/ws_bytes.
 *   - The scratch it needs (about 2.3 MiB: split-K partials, the normalized low-rank query,
 *     an error word) is one fixed array inside the library, reserved on every GPU that loads
 *     the library until the process exits. No call allocates or frees anything.
 *   - batch > MFA_NOALLOC_MAX_BATCH returns MFA_ERR_WORKSPACE (the built-in scratch is too
 *     small for it); batch < 1, eps <= 0 or a null/misaligned pointer return
 *     MFA_ERR_INVALID_ARG. Nothing is enqueued in either case.
 *   - The first call on a device looks up the array's device address on that device (it
 *     must be the current device) and keeps it for the rest of the process; make that first
 *     call before any stream capture. A device reset (cudaDeviceReset) unloads the array, so
 *     this call must not be used on that device again afterwards.
 *   - Every call on a device uses the same array, which keeps the last call's contents.
 *     Calls that can run at the same time on the GPU (unordered streams, several host
 *     threads) race on it and corrupt each other's results: order them on one stream.
 *   - Device-side errors (a bounded wait that expired) set bits in the array's error word,
 *     which stays set across calls until mfa_query_proj_noalloc_get_error reads it. */
MFA_API mfa_status mfa_query_proj_noalloc(const void* x, const void* w_qdown, const void* gamma,
                                          const void* w_qup, float eps, void* q_out,
                                          int32_t batch, void* stream);

/* The device-side status of mfa_query_proj_noalloc on the current device: synchronizes
 * `stream`, then returns and clears the error word of the built-in scratch (MFA_OK,
 * or MFA_ERR_TIMEOUT if a bounded wait expired in a call since the last read). It allocates
 * nothing. Like the calls it reports on, it must not overlap them on another stream. */
MFA_API mfa_status mfa_query_proj_noalloc_get_error(void* stream);

/* Diagnostic for mfa_query_proj_noalloc_get_error (no counterpart on the Step-3 pages):
 * enqueues the kernel of mfa_wait_selftest on the built-in scratch's error word, so that
 * the next mfa_query_proj_noalloc_get_error returns MFA_ERR_TIMEOUT. limit_us as for
 * mfa_wait_selftest (1 .. 1,000,000; otherwise MFA_ERR_INVALID_ARG, nothing enqueued). */
MFA_API mfa_status mfa_query_proj_noalloc_wait_selftest(uint32_t limit_us, void* stream);

/* ---------------------------------------------------------------------------------------
 * Diagnostics
 * ------------------------------------------------------------------------------------- */

/* Check of the failure detection the compute calls rely on (the Step-3 pages have no
 * counterpart: it tests the library, not the method). Every wait inside the library's
 * kernels is bounded: when one expires, the kernel stops, drains what it started and sets
 * MFA_ERR_TIMEOUT in the workspace. This call enqueues one small kernel that makes exactly
 * such a wait on a barrier nothing ever completes, with a limit of `limit_us` microseconds
 * (1 .. 1,000,000) instead of the compute calls' 2 s.
 *   ws: a workspace (mfa_workspace_bytes(b) for any b, initialized); only its error word is
 *   touched. After the stream reaches the kernel's end, mfa_get_error(ws) returns
 *   MFA_ERR_TIMEOUT, and the device and `ws` remain usable by every other call.
 *   Returns MFA_ERR_INVALID_ARG for a null or misaligned ws, ws_bytes < 256 or a limit out
 *   of range (nothing enqueued), MFA_ERR_CUDA if the launch fails. */
MFA_API mfa_status mfa_wait_selftest(void* ws, size_t ws_bytes, uint32_t limit_us,
                                     void* stream);

/* The length-aware split plan of the decode attention (the scheduler that balances the K/V
 * stream over the persistent grid; see mfa_decode_attn), as the device builds it for the
 * lengths in `seq_lens` (device int32 [kv->batch]) and the capacities in kv's table, for a
 * grid of `grid` CTAs (1 .. 256; the attention itself uses one CTA per SM). The plan cuts
 * every accepted sequence (1 <= length <= capacity) into tiles of 128 positions, lays them
 * end to end and gives CTA g the tiles [g NT / G, (g + 1) NT / G), G = min(grid, NT); the part
 * of a sequence inside one CTA's range is a work item. Rejected sequences have no items.
 *   out: device int32 buffer of at least 3 + 8 (grid + batch) entries, written as
 *     out[0] = G, out[1] = NT, out[2] = n (work items), then item i at out[3 + 8 i]:
 *     (cta, sequence, first position, one past the last, partial slot or -1 when the
 *     sequence is finished by this item alone, CTAs sharing the sequence, this item's index
 *     among them, 0). Items are listed CTA by CTA, each CTA's in the order it streams them.
 *   Returns MFA_ERR_INVALID_ARG (null or misaligned pointer, batch or grid out of range),
 *   MFA_ERR_WORKSPACE (out too small), MFA_ERR_CUDA (launch failure); asynchronous on
 *   `stream` otherwise. */
MFA_API mfa_status mfa_split_plan(const mfa_kv_cache* kv, const int32_t* seq_lens,
                                  int32_t grid, int32_t* out, size_t out_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Captured decode steps (no counterpart in the pages: a host-cost option of this library)
 * ------------------------------------------------------------------------------------- */

/* One decode step captured once as a CUDA graph on the current device, for callers whose
 * host thread, not the GPU, paces the loop: replaying it costs one graph launch instead of
 * the step's five or six kernel launches. A replay runs exactly the launches that
 * mfa_decode_layer (w8: mfa_decode_layer_w8) would make with these arguments, so its results
 * are bit-identical to that call's. The arguments are read once, at capture: the addresses
 * and the mfa_kv_cache fields must stay valid and unchanged for the handle's life, while the
 * buffers' contents (x, seq_lens, the weights, the cache rows, the KV table's entries) may
 * change between replays. A replay begins only after the stream's earlier work has
 * completed (no programmatic overlap with the kernel before it), so back-to-back direct
 * calls, which do overlap, are the faster choice whenever the GPU paces the loop.
 *   *out receives the handle (NULL on error). Errors as mfa_decode_layer, plus
 *   MFA_ERR_CUDA if the capture or the graph instantiation fails. The capture runs on a
 *   stream of the library's own and does not touch the caller's streams. */
typedef struct mfa_step_graph mfa_step_graph;

MFA_API mfa_status mfa_decode_layer_graph(const void* x, const void* w_qdown, const void* gamma,
                                          const void* w_qup, const void* w_k, const void* w_v,
                                          float eps, const mfa_kv_cache* kv,
                                          const int32_t* seq_lens, float scale, void* q_out,
                                          void* out, void* ws, size_t ws_bytes,
                                          mfa_step_graph** graph);

MFA_API mfa_status mfa_decode_layer_w8_graph(const void* x, mfa_w8 w_qdown, const void* gamma,
                                             mfa_w8 w_qup, mfa_w8 w_k, mfa_w8 w_v, float eps,
                                             const mfa_kv_cache* kv, const int32_t* seq_lens,
                                             float scale, void* q_out, void* out, void* ws,
                                             size_t ws_bytes, mfa_step_graph** graph);

/* Replay a captured step on `stream` (a stream of the device it was captured on).
 * MFA_ERR_INVALID_ARG for a NULL handle, MFA_ERR_CUDA if the launch fails. */
MFA_API mfa_status mfa_step_graph_launch(const mfa_step_graph* graph, void* stream);

/* Release a handle (NULL is ignored). Replays already enqueued still run: the graph is
 * freed once they complete. */
MFA_API void mfa_step_graph_destroy(mfa_step_graph* graph);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MFA_H_ */
