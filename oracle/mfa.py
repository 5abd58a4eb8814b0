"""One decode step of Step-3's MFA attention layer, float64 (test infrastructure only).

Source passages (Step-3 pages):

* bud-325 summary, "Key claims" and "Method": hidden size 7168; the query is produced by a
  low-rank factorization -- down-projected from 7168 to rank 2048, normalized, then
  up-projected to 64 heads x 256; one K head and one V head (head dim 256) are shared by
  all 64 query heads, so the KV cache holds one K and one V vector per token; per-token
  decode attention cost is max(attention compute, KV memory access).
* redeep.blog post, "What's New" (same factorization: 7168 -> 2048 -> norm -> 64 x 256) and
  the architecture table (hidden 7168, low-rank query dimension 2048, 64 query heads,
  head dimension 256, max context 65,536).

Readings where the pages are silent (each one is listed with its reason in the design
notes of the repository):

* the "normalization" is RMSNorm over the 2048-wide vector, eps = 1e-6 inside the square
  root, elementwise gain gamma, no bias;
* no positional encoding; q, k, v are used as projected;
* k = x W_k and v = x W_v, each [7168, 256], straight from the hidden state;
* softmax scale 1/sqrt(256) = 1/16;
* weights are row-major [in, out]; head h of the up-projection is output columns
  [256 h, 256 h + 256);
* ``seq_lens[b]`` counts the positions attended *after* the new token is appended; the new
  token's K/V row is written at row ``seq_lens[b] - 1`` and attended to;
* the FP8 KV cache stores e4m3(value / scale) with one float32 scale per tensor for K and
  one for V; bf16 caches store bf16(value); every rounding is to nearest, ties to even.

The method reaches exactly (up to rounding order) the plain definition of attention, so
the oracle is that definition: scores, a max-subtracted softmax and a weighted sum, with
numpy's float64 matmul as the only library step.
"""

import numpy as np

from . import codecs

# Layer dimensions stated on the pages (bud-325 "Key claims"; redeep architecture table).
HIDDEN = 7168
Q_RANK = 2048
N_HEADS = 64
HEAD_DIM = 256
MAX_CONTEXT = 65536

# Readings for what the pages leave open.
RMS_EPS = 1e-6
SOFTMAX_SCALE = 1.0 / 16.0  # 1 / sqrt(HEAD_DIM)

KV_BF16 = "bf16"
KV_FP8 = "fp8_e4m3"


# ----------------------------------------------------------------------------------------
# query path: x -> down-projection -> normalization -> up-projection -> 64 heads
# ----------------------------------------------------------------------------------------


def q_down(x, w_qdown):
    """c = x W_qdown: the low-rank query down-projection (7168 -> 2048).

    x [B, D], w_qdown [D, R] (float64 values) -> c [B, R].
    Pinned by: small-integer inputs whose sums are exact, compared with exact Python
    integer sums (tests/test_oracle_mfa.py)."""
    return np.asarray(x, np.float64) @ np.asarray(w_qdown, np.float64)


def rms_norm(c, gamma, eps=RMS_EPS):
    """c_hat = c / sqrt(mean(c^2) + eps) * gamma over the last axis (the "normalized" step,
    read as RMSNorm).

    Pinned by: the closed form mean(c_hat^2) = m / (m + eps) for gamma = 1 (m = mean(c^2)),
    sign preservation, scale invariance and a hand-worked vector."""
    c = np.asarray(c, np.float64)
    ms = np.mean(c * c, axis=-1, keepdims=True)
    return c / np.sqrt(ms + eps) * np.asarray(gamma, np.float64)


def q_up(c_hat, w_qup, n_heads=N_HEADS):
    """q = c_hat W_qup reshaped to [B, n_heads, head_dim]; head h is output columns
    [h * head_dim, (h + 1) * head_dim).

    Pinned by: exact small-integer sums and a one-hot weight that routes a chosen input
    element to a chosen (head, dim) slot."""
    q = np.asarray(c_hat, np.float64) @ np.asarray(w_qup, np.float64)
    b, n = q.shape
    return q.reshape(b, n_heads, n // n_heads)


def query_proj(x, w_qdown, gamma, w_qup, eps=RMS_EPS, n_heads=N_HEADS, emulate=True):
    """The MFA query path. Returns (c_hat, q).

    With ``emulate`` the two results that the CUDA path stores as bf16 buffers (the
    normalized low-rank query that feeds the up-projection, and q itself) are rounded to
    bf16 here as well, so the end-to-end comparison measures the kernels' arithmetic
    rather than those two storage roundings. ``emulate=False`` keeps pure float64."""
    c_hat = rms_norm(q_down(x, w_qdown), gamma, eps)
    if emulate:
        c_hat = codecs.bf16_round(c_hat)
    q = q_up(c_hat, w_qup, n_heads)
    if emulate:
        q = codecs.bf16_round(q)
    return c_hat, q


# ----------------------------------------------------------------------------------------
# the shared K/V head and its cache
# ----------------------------------------------------------------------------------------


def kv_project(x, w_k, w_v):
    """k = x W_k, v = x W_v: the single shared K head and V head of the new token.

    Pinned by: one-hot weights (k equals a chosen element of x exactly)."""
    x = np.asarray(x, np.float64)
    return x @ np.asarray(w_k, np.float64), x @ np.asarray(w_v, np.float64)


def kv_store(values, kv_dtype, scale=1.0):
    """Values -> the codes a cache of ``kv_dtype`` holds: bf16 bits (uint16), or
    e4m3(value / scale) codes (uint8)."""
    if kv_dtype == KV_BF16:
        return codecs.bf16_encode(values)
    if kv_dtype == KV_FP8:
        return codecs.e4m3_encode(np.asarray(values, np.float64) / float(scale))
    raise ValueError(f"unknown kv dtype {kv_dtype!r}")


def kv_load(codes, kv_dtype, scale=1.0):
    """Cache codes -> float64 values (e4m3 codes are multiplied by their scale)."""
    if kv_dtype == KV_BF16:
        return codecs.bf16_decode(codes)
    if kv_dtype == KV_FP8:
        return codecs.e4m3_decode(codes) * float(scale)
    raise ValueError(f"unknown kv dtype {kv_dtype!r}")


def kv_gather_paged(pool, page_ids, n_rows, page_size):
    """Rows [0, n_rows) of one sequence of a paged cache: row j is row j % page_size of page
    page_ids[j // page_size] of ``pool`` [num_pages, page_size, d] (the page-table layout of
    the serving engines the step3-fp8 model page deploys with, vLLM and SGLang). Returns the
    codes [n_rows, d].

    Pinned by: a contiguous cache cut into pages placed at shuffled pool slots gathers back
    to itself; rows past n_rows and pages outside the list are never read."""
    rows = [pool[int(page_ids[j // page_size])][j % page_size] for j in range(int(n_rows))]
    if not rows:
        return np.zeros((0,) + tuple(np.shape(pool)[2:]), dtype=np.asarray(pool).dtype)
    return np.stack(rows)


def kv_append(k_cache, v_cache, pos, k_codes, v_codes):
    """Write the new token's K/V codes at row ``pos[b]`` of sequence b's cache.

    k_cache, v_cache: lists of per-sequence code arrays [cap_b, head_dim]. Returns new
    lists; every other row is left as it was. Pinned by: exact byte comparison of every
    row (tests/test_oracle_mfa.py)."""
    k_out, v_out = [], []
    for b in range(len(k_cache)):
        kc = np.array(k_cache[b], copy=True)
        vc = np.array(v_cache[b], copy=True)
        p = int(pos[b])
        if not 0 <= p < kc.shape[0]:
            raise IndexError(f"sequence {b}: row {p} outside capacity {kc.shape[0]}")
        kc[p] = k_codes[b]
        vc[p] = v_codes[b]
        k_out.append(kc)
        v_out.append(vc)
    return k_out, v_out


# ----------------------------------------------------------------------------------------
# attention of the 64 query heads over the shared K/V head
# ----------------------------------------------------------------------------------------


def attention_weights(q_b, keys, scale=SOFTMAX_SCALE):
    """Softmax weights of one sequence: w[h, j] = exp(s[h, j]) / sum_j exp(s[h, j]) with
    s[h, j] = scale * q_b[h] . keys[j]. q_b [H, d], keys [L, d] -> [H, L].

    The maximum over j is subtracted before exp, which leaves the weights unchanged.
    Pinned by: two-token closed form (logistic of the score difference), weights summing
    to 1, permutation invariance, and pure-Python brute force."""
    s = (np.asarray(q_b, np.float64) @ np.asarray(keys, np.float64).T) * scale
    s = s - np.max(s, axis=1, keepdims=True)
    e = np.exp(s)
    return e / np.sum(e, axis=1, keepdims=True)


def decode_attn_seq(q_b, keys, values, scale=SOFTMAX_SCALE):
    """out[h] = sum_j w[h, j] values[j] for one sequence. q_b [H, d], keys/values [L, d]
    (float64, L >= 1) -> [H, d].

    Pinned by: L = 1 gives out = v; identical keys, or q = 0, give the mean of V;
    brute force at tiny sizes."""
    if keys.shape[0] < 1:
        raise ValueError("attention needs at least one cached position")
    return attention_weights(q_b, keys, scale) @ np.asarray(values, np.float64)


def decode_attn(q, k_cache, v_cache, seq_lens, kv_dtype=KV_BF16, k_scale=1.0, v_scale=1.0,
                scale=SOFTMAX_SCALE, seqs=None):
    """Attention of every sequence (or of the sequences listed in ``seqs``) over rows
    [0, seq_lens[b]) of its cache codes. q [B, H, d] float64 -> out [len(seqs), H, d]."""
    seqs = range(len(k_cache)) if seqs is None else seqs
    out = []
    for b in seqs:
        n = int(seq_lens[b])
        keys = kv_load(k_cache[b][:n], kv_dtype, k_scale)
        vals = kv_load(v_cache[b][:n], kv_dtype, v_scale)
        out.append(decode_attn_seq(q[b], keys, vals, scale))
    return np.stack(out)


# ----------------------------------------------------------------------------------------
# the whole decode step
# ----------------------------------------------------------------------------------------


def decode_layer(x, w_qdown, gamma, w_qup, w_k, w_v, k_cache, v_cache, seq_lens,
                 kv_dtype=KV_BF16, k_scale=1.0, v_scale=1.0, eps=RMS_EPS,
                 scale=SOFTMAX_SCALE, n_heads=N_HEADS, emulate=True, seqs=None):
    """One MFA decode step, in the order the pages state it: the query path, then the new
    token's K/V appended to its sequence's cache at row seq_lens[b] - 1, then attention of
    all heads over rows [0, seq_lens[b]).

    Returns a dict with c_hat, q, k_codes, v_codes (the appended rows), k_cache, v_cache
    (after the append) and out [B or len(seqs), H, d]."""
    c_hat, q = query_proj(x, w_qdown, gamma, w_qup, eps, n_heads, emulate)
    k_new, v_new = kv_project(x, w_k, w_v)
    k_codes = kv_store(k_new, kv_dtype, k_scale)
    v_codes = kv_store(v_new, kv_dtype, v_scale)
    pos = [int(n) - 1 for n in seq_lens]
    k_cache2, v_cache2 = kv_append(k_cache, v_cache, pos, k_codes, v_codes)
    out = decode_attn(q, k_cache2, v_cache2, seq_lens, kv_dtype, k_scale, v_scale, scale,
                      seqs)
    return dict(c_hat=c_hat, q=q, k_codes=k_codes, v_codes=v_codes, k_cache=k_cache2,
                v_cache=v_cache2, out=out)


# ----------------------------------------------------------------------------------------
# the attention side of a decode step: output projection and a stack of layers
# ----------------------------------------------------------------------------------------

O_WIDTH = N_HEADS * HEAD_DIM  # 16384: the 64 heads' outputs of one token, concatenated


def o_proj(out, w_o):
    """y = out W_o: the attention output of all heads, [B, H, d] or [B, H * d], projected
    back to the hidden width (bud-325 "Method": the per-token cost counts the linear
    projections around attention, and the layer hands a hidden-width vector on to the FFN;
    the [16384, 7168] shape of W_o is the reading that the 64 x 256 head outputs return to
    hidden size 7168). Float64.

    Pinned by: small-integer inputs against a brute-force triple loop, and a one-hot W_o
    that copies chosen columns of out."""
    o = np.asarray(out, np.float64)
    o = o.reshape(o.shape[0], -1)
    return o @ np.asarray(w_o, np.float64)


def attention_side_step(x, layers, seq_lens, kv_dtype=KV_BF16, eps=RMS_EPS,
                        scale=SOFTMAX_SCALE, n_heads=N_HEADS, emulate=True):
    """The attention side of one decode step through a stack of layers. Each entry of
    ``layers`` is a dict with w_qdown, gamma, w_qup, w_k, w_v, w_o, k_cache, v_cache,
    k_scale, v_scale. Layer l runs decode_layer on its hidden input, projects the attention
    output with its W_o, and the result is layer l + 1's hidden input: under Attention-FFN
    Disaggregation (bud-325 "Key claims") the FFN runs on other GPUs and its result comes
    back as the next layer's input, so with the FFN out of scope the projection is handed
    on directly. With ``emulate`` the bf16 tensors the GPU path stores between calls (the
    attention output and y) are rounded to bf16 as it does.

    Returns (per-layer list of decode_layer results, each with y added; the last y)."""
    results = []
    h = np.asarray(x, np.float64)
    for lay in layers:
        r = decode_layer(h, lay["w_qdown"], lay["gamma"], lay["w_qup"], lay["w_k"],
                         lay["w_v"], lay["k_cache"], lay["v_cache"], seq_lens, kv_dtype,
                         lay.get("k_scale", 1.0), lay.get("v_scale", 1.0), eps, scale,
                         n_heads, emulate=emulate)
        out = codecs.bf16_round(r["out"]) if emulate else r["out"]
        y = o_proj(out, lay["w_o"])
        if emulate:
            y = codecs.bf16_round(y)
        r["y"] = y
        results.append(r)
        h = y
    return results, h


# ----------------------------------------------------------------------------------------
# FP8 projections: block-FP8 weights (the step3-fp8 model page: checkpoints in bf16 and
# block-fp8) and FP8 activations (the Step-3 pages: the whole model runs in FP8, bud-325
# "Key claims")
# ----------------------------------------------------------------------------------------

W8_BLOCK = 128  # reading: one float32 scale per 128 x 128 block of a weight
A8_GROUP = 128  # reading: one float32 scale per 128 consecutive values of an activation row


def w8_dequantize(codes, scales, block=W8_BLOCK):
    """A block-FP8 weight as real values: ``codes`` [out, in] uint8 are e4m3 codes in the
    checkpoints' [out, in] order, ``scales`` [ceil(out / block), ceil(in / block)] float32;
    weight[o, i] = code[o, i] * scale[o // block, i // block], exactly. Returns float64
    [in, out] (the [in, out] order of the other projections). The page names the format
    without a block size; 128 x 128 is the reading taken.

    Pinned by: power-of-two scales placed per block and ragged edge blocks, against
    code * scale element by element."""
    c = codecs.e4m3_decode(np.asarray(codes))
    s = np.asarray(scales, np.float64)
    s_full = np.repeat(np.repeat(s, block, axis=0), block, axis=1)[:c.shape[0], :c.shape[1]]
    return (c * s_full).T


def a8_quantize(a, group=A8_GROUP):
    """An activation [rows, n] (bf16 values) in FP8: per row and group of ``group``
    consecutive values, scale = max |a| / 448 (1 for an all-zero group) and code =
    e4m3(a / scale), round to nearest even, saturating. The scale and the quotient are
    float32 operations (round to nearest even), so both sides of a comparison decide each
    code in the same precision. Returns (codes uint8 [rows, n], scales float32
    [rows, ceil(n / group)]).

    Pinned by: a group whose max is a power of two times 448 (exact scale and codes), the
    max element always coding to +-448, zero groups, and brute force on small rows."""
    a = np.asarray(a, np.float64)
    rows, n = a.shape
    ng = -(-n // group)
    codes = np.zeros((rows, n), np.uint8)
    scales = np.ones((rows, ng), np.float32)
    for g in range(ng):
        blk = a[:, g * group:(g + 1) * group].astype(np.float32)
        amax = np.abs(blk).max(axis=1)
        sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        q = (blk / sc[:, None]).astype(np.float32)
        codes[:, g * group:(g + 1) * group] = codecs.e4m3_encode(q.astype(np.float64))
        scales[:, g] = sc
    return codes, scales


def a8_dequantize(codes, scales, group=A8_GROUP):
    """codes [rows, n] and scales [rows, ceil(n / group)] -> float64 values, exactly."""
    c = codecs.e4m3_decode(np.asarray(codes))
    s = np.repeat(np.asarray(scales, np.float64), group, axis=1)[:, :c.shape[1]]
    return c * s


def fp8_project(a, w_codes, w_scales):
    """A projection on the FP8 path: the activation rows quantized by ``a8_quantize``, the
    weight block-FP8; the products of the real values, summed in float64. Returns [rows,
    out].

    Pinned by: ``math.fsum`` of the decoded codes times their scales, element by element."""
    ac, asc = a8_quantize(a)
    return a8_dequantize(ac, asc) @ w8_dequantize(w_codes, w_scales)


def query_proj_fp8(x, wq_codes, wq_scales, gamma, wu_codes, wu_scales, eps=RMS_EPS,
                   n_heads=N_HEADS, emulate=True):
    """The query path on the FP8 path: c = fp8_project(x, W_qdown), RMSNorm as ever, then
    q = fp8_project(c_hat, W_qup) (c_hat rounded to bf16 first with ``emulate``, as stored).
    Returns (c_hat, q).

    Pinned by: a pure-Python brute force of the whole chain at small sizes (exact ``fsum``
    sums of decoded codes times block scales, the bf16 rounding of c_hat before it is
    quantized, head-major output columns), one-hot routing of chosen inputs to chosen
    (head, dim) slots, and two planted mistakes (quantizing c_hat before its bf16 rounding;
    a dim-major reshape) that the brute force rejects."""
    c_hat = rms_norm(fp8_project(x, wq_codes, wq_scales), gamma, eps)
    if emulate:
        c_hat = codecs.bf16_round(c_hat)
    q = fp8_project(c_hat, wu_codes, wu_scales)
    b, n = q.shape
    q = q.reshape(b, n_heads, n // n_heads)
    if emulate:
        q = codecs.bf16_round(q)
    return c_hat, q
