"""Pins of the float64 oracle of the MFA decode step against things other than itself:
exact integer arithmetic, closed forms, invariants the definition fixes, pure-Python brute
force at tiny sizes, the page-stated dimensions, and planted mistakes that must be caught."""

import json
import math
import os

import numpy as np
import pytest

from oracle import codecs
from oracle import mfa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_constants_match_page_dimensions():
    with open(os.path.join(GOLDEN, "page_dims.json")) as f:
        dims = json.load(f)
    assert mfa.HIDDEN == dims["hidden"]
    assert mfa.Q_RANK == dims["q_rank"]
    assert mfa.N_HEADS == dims["n_heads"]
    assert mfa.HEAD_DIM == dims["head_dim"]
    assert mfa.MAX_CONTEXT == dims["max_context"]
    assert mfa.SOFTMAX_SCALE == 1.0 / math.sqrt(dims["head_dim"])


# ----------------------------------------------------------------------------------------
# projections: exact small-integer arithmetic against Python integers
# ----------------------------------------------------------------------------------------


def _int_matmul(a, b):
    return [[sum(int(a[i][k]) * int(b[k][j]) for k in range(len(b))) for j in range(len(b[0]))]
            for i in range(len(a))]


@pytest.mark.parametrize("bsz,din,dout", [(1, 7, 5), (3, 16, 12), (2, 33, 8)])
def test_projections_exact_on_small_integers(bsz, din, dout):
    rng = np.random.default_rng(din)
    x = rng.integers(-3, 4, (bsz, din))
    w = rng.integers(-2, 3, (din, dout))
    want = np.array(_int_matmul(x.tolist(), w.tolist()), dtype=np.float64)
    assert np.array_equal(mfa.q_down(x, w), want)
    k, v = mfa.kv_project(x, w, -w)
    assert np.array_equal(k, want) and np.array_equal(v, -want)
    q = mfa.q_up(x, w, n_heads=1)
    assert np.array_equal(q.reshape(bsz, dout), want)


def test_q_up_head_ordering_one_hot():
    # W routes input element i to output column 256 h + j: head h, dim j
    r, heads, d = 6, 4, 8
    rng = np.random.default_rng(0)
    for _ in range(10):
        i, h, j = rng.integers(r), rng.integers(heads), rng.integers(d)
        w = np.zeros((r, heads * d))
        w[i, h * d + j] = 1.0
        c = rng.standard_normal((2, r))
        q = mfa.q_up(c, w, n_heads=heads)
        expect = np.zeros((2, heads, d))
        expect[:, h, j] = c[:, i]
        assert np.array_equal(q, expect)


# ----------------------------------------------------------------------------------------
# normalization
# ----------------------------------------------------------------------------------------


def test_rms_norm_hand_worked():
    # c = (3, 4): mean square 12.5; with eps = 0 the result is c / sqrt(12.5)
    out = mfa.rms_norm(np.array([[3.0, 4.0]]), np.ones(2), eps=0.0)
    assert np.allclose(out, [[3 / math.sqrt(12.5), 4 / math.sqrt(12.5)]], rtol=0, atol=1e-15)
    out = mfa.rms_norm(np.array([[3.0, 4.0]]), np.array([2.0, -1.0]), eps=0.0)
    assert np.allclose(out, [[6 / math.sqrt(12.5), -4 / math.sqrt(12.5)]], rtol=0, atol=1e-15)


@pytest.mark.parametrize("scale", [1e-4, 1e-2, 1.0, 37.0])
def test_rms_norm_closed_form_mean_square(scale):
    rng = np.random.default_rng(1)
    c = rng.standard_normal((5, 2048)) * scale
    eps = 1e-6
    out = mfa.rms_norm(c, np.ones(2048), eps)
    m = np.mean(c * c, axis=-1)
    assert np.allclose(np.mean(out * out, axis=-1), m / (m + eps), rtol=1e-12, atol=0)
    assert np.array_equal(np.sign(out), np.sign(c))


# ----------------------------------------------------------------------------------------
# attention: closed forms, invariants, brute force
# ----------------------------------------------------------------------------------------


def test_attention_single_position_returns_v():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((64, 256)) * 5
    k = rng.standard_normal((1, 256))
    v = rng.standard_normal((1, 256))
    out = mfa.decode_attn_seq(q, k, v)
    assert np.array_equal(out, np.repeat(v, 64, axis=0))


def test_attention_two_positions_closed_form_ln3():
    # q . k0 / 16 = ln 3 and q . k1 = 0  =>  weights 3/4 and 1/4 exactly (logistic)
    d = 256
    q = np.zeros((1, d))
    q[0, 0] = 16.0
    k = np.zeros((2, d))
    k[0, 0] = math.log(3.0)
    v = np.stack([np.full(d, 1.0), np.full(d, 5.0)])
    out = mfa.decode_attn_seq(q, k, v)
    assert np.allclose(out, 0.75 * v[0] + 0.25 * v[1], rtol=0, atol=1e-14)
    w = mfa.attention_weights(q, k)
    assert np.allclose(w, [[0.75, 0.25]], rtol=0, atol=1e-15)


def test_attention_logistic_for_random_pairs():
    rng = np.random.default_rng(3)
    for _ in range(20):
        q = rng.standard_normal((3, 256))
        k = rng.standard_normal((2, 256)) * 3
        w = mfa.attention_weights(q, k)
        s = q @ k.T / 16.0
        w0 = 1.0 / (1.0 + np.exp(s[:, 1] - s[:, 0]))
        assert np.allclose(w[:, 0], w0, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("L", [1, 2, 5, 64, 129])
def test_attention_identical_keys_or_zero_query_give_mean_of_v(L):
    rng = np.random.default_rng(L)
    q = rng.standard_normal((64, 256)) * 4
    v = rng.standard_normal((L, 256))
    k_same = np.repeat(rng.standard_normal((1, 256)), L, axis=0)
    mean_v = np.mean(v, axis=0)
    assert np.allclose(mfa.decode_attn_seq(q, k_same, v), mean_v, rtol=0, atol=1e-13)
    k = rng.standard_normal((L, 256))
    assert np.allclose(mfa.decode_attn_seq(np.zeros((64, 256)), k, v), mean_v, rtol=0,
                       atol=1e-13)


def test_attention_weights_sum_to_one_and_permutation_invariance():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((64, 256)) * 2
    k = rng.standard_normal((300, 256)) * 2
    v = rng.standard_normal((300, 256))
    w = mfa.attention_weights(q, k)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    assert (w >= 0).all()
    perm = rng.permutation(300)
    assert np.allclose(mfa.decode_attn_seq(q, k, v), mfa.decode_attn_seq(q, k[perm], v[perm]),
                       rtol=1e-12, atol=1e-14)
    # heads are independent: identical query rows give identical output rows
    q2 = np.repeat(q[:1], 64, axis=0)
    o = mfa.decode_attn_seq(q2, k, v)
    assert np.allclose(o, np.repeat(o[:1], 64, axis=0), rtol=0, atol=0)


def _brute_layer(x, wd, gamma, wu, wk, wv, caches_k, caches_v, lens, heads, eps, scale):
    """Pure-Python loops (math.fsum / math.exp / math.sqrt) of the whole step, no numpy."""
    bsz, dim = len(x), len(x[0])
    rank, hd = len(wd[0]), len(wk[0])
    hdim = len(wu[0]) // heads
    outs = []
    for b in range(bsz):
        c = [math.fsum(x[b][i] * wd[i][r] for i in range(dim)) for r in range(rank)]
        ms = math.fsum(t * t for t in c) / rank
        ch = [c[r] / math.sqrt(ms + eps) * gamma[r] for r in range(rank)]
        q = [math.fsum(ch[r] * wu[r][j] for r in range(rank)) for j in range(heads * hdim)]
        kn = [math.fsum(x[b][i] * wk[i][j] for i in range(dim)) for j in range(hd)]
        vn = [math.fsum(x[b][i] * wv[i][j] for i in range(dim)) for j in range(hd)]
        n = lens[b]
        # caches_* already hold the new row, rounded to bf16 by the cache, at row n - 1;
        # it must lie within half a bf16 ulp (<= 2**-8 relative) of the exact projection
        for new, row in ((kn, caches_k[b][n - 1]), (vn, caches_v[b][n - 1])):
            for a, r in zip(new, row):
                assert abs(a - r) <= abs(a) * 2.0 ** -8
        ks = [list(r) for r in caches_k[b][:n]]
        vs = [list(r) for r in caches_v[b][:n]]
        head_out = []
        for h in range(heads):
            qh = q[h * hdim:(h + 1) * hdim]
            s = [scale * math.fsum(qh[j] * ks[t][j] for j in range(hd)) for t in range(n)]
            m = max(s)
            e = [math.exp(si - m) for si in s]
            z = math.fsum(e)
            head_out.append([math.fsum(e[t] * vs[t][j] for t in range(n)) / z
                             for j in range(hd)])
        outs.append(head_out)
    return np.array(outs)


@pytest.mark.parametrize("lens", [[1], [3, 1, 7], [9, 4]])
def test_decode_layer_matches_pure_python_brute_force(lens):
    rng = np.random.default_rng(sum(lens))
    dim, rank, heads, hd = 12, 8, 4, 6
    bsz = len(lens)
    x = rng.standard_normal((bsz, dim))
    wd = rng.standard_normal((dim, rank)) / math.sqrt(dim)
    gamma = rng.uniform(0.5, 1.5, rank)
    wu = rng.standard_normal((rank, heads * hd)) / math.sqrt(rank)
    wk = rng.standard_normal((dim, hd)) / math.sqrt(dim)
    wv = rng.standard_normal((dim, hd)) / math.sqrt(dim)
    ck = [rng.standard_normal((n, hd)) for n in lens]
    cv = [rng.standard_normal((n, hd)) for n in lens]
    eps, scale = 1e-6, 1.0 / math.sqrt(hd)
    # the oracle works on stored codes; use bf16-exact values so the codes are lossless
    ck = [codecs.bf16_round(t) for t in ck]
    cv = [codecs.bf16_round(t) for t in cv]
    kc = [codecs.bf16_encode(t) for t in ck]
    vc = [codecs.bf16_encode(t) for t in cv]
    res = mfa.decode_layer(x, wd, gamma, wu, wk, wv, kc, vc, lens, eps=eps, scale=scale,
                           n_heads=heads, emulate=False)
    # the appended row is rounded to bf16 by the cache; feed brute force the same row
    k_new, v_new = mfa.kv_project(x, wk, wv)
    ck2 = [np.vstack([ck[b][:lens[b] - 1], codecs.bf16_round(k_new[b])[None]])
           for b in range(bsz)]
    cv2 = [np.vstack([cv[b][:lens[b] - 1], codecs.bf16_round(v_new[b])[None]])
           for b in range(bsz)]
    want = _brute_layer(x.tolist(), wd.tolist(), gamma.tolist(), wu.tolist(), wk.tolist(),
                        wv.tolist(), [t.tolist() for t in ck2], [t.tolist() for t in cv2],
                        lens, heads, eps, scale)
    assert np.allclose(res["out"], want, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------------------
# KV append: bytes
# ----------------------------------------------------------------------------------------


@pytest.mark.parametrize("kv_dtype", [mfa.KV_BF16, mfa.KV_FP8])
def test_kv_append_writes_exactly_one_row(kv_dtype):
    rng = np.random.default_rng(9)
    caps = [5, 1, 8]
    dt = np.uint16 if kv_dtype == mfa.KV_BF16 else np.uint8
    kc = [rng.integers(0, 120, (c, 16)).astype(dt) for c in caps]
    vc = [rng.integers(0, 120, (c, 16)).astype(dt) for c in caps]
    pos = [4, 0, 3]
    newk = rng.integers(0, 120, (3, 16)).astype(dt)
    newv = rng.integers(0, 120, (3, 16)).astype(dt)
    k2, v2 = mfa.kv_append(kc, vc, pos, newk, newv)
    for b, p in enumerate(pos):
        for r in range(caps[b]):
            wk = newk[b] if r == p else kc[b][r]
            wv = newv[b] if r == p else vc[b][r]
            assert np.array_equal(k2[b][r], wk) and np.array_equal(v2[b][r], wv)
        assert np.array_equal(kc[b], kc[b])  # inputs untouched
    with pytest.raises(IndexError):
        mfa.kv_append(kc, vc, [5, 0, 0], newk, newv)


def test_kv_store_fp8_power_of_two_scale_is_exact():
    # one-hot projection -> k equals a chosen element of x; values on the e4m3 grid times a
    # power-of-two scale are stored and loaded back exactly
    grid = codecs.e4m3_decode(np.arange(0, 0x7F))
    rng = np.random.default_rng(12)
    vals = rng.choice(grid, 64) * 0.125 * rng.choice([-1, 1], 64)
    x = vals[None, :]
    w = np.eye(64)
    k, v = mfa.kv_project(x, w, 2 * w)
    codes = mfa.kv_store(k, mfa.KV_FP8, 0.125)
    assert np.array_equal(mfa.kv_load(codes, mfa.KV_FP8, 0.125), vals[None, :])
    codes = mfa.kv_store(v, mfa.KV_FP8, 0.25)
    assert np.array_equal(mfa.kv_load(codes, mfa.KV_FP8, 0.25), 2 * vals[None, :])


def test_decode_layer_appends_at_len_minus_one_and_attends_to_it():
    # L = 1: the only attended row is the new token's v (rounded to bf16), for every head
    rng = np.random.default_rng(13)
    dim, rank, heads, hd = 10, 4, 3, 5
    x = rng.standard_normal((2, dim))
    wd, wu = rng.standard_normal((dim, rank)), rng.standard_normal((rank, heads * hd))
    wk, wv = rng.standard_normal((dim, hd)), rng.standard_normal((dim, hd))
    kc = [codecs.bf16_encode(rng.standard_normal((4, hd))) for _ in range(2)]
    vc = [codecs.bf16_encode(rng.standard_normal((4, hd))) for _ in range(2)]
    res = mfa.decode_layer(x, wd, np.ones(rank), wu, wk, wv, kc, vc, [1, 3], n_heads=heads,
                           scale=0.3)
    v_new = codecs.bf16_round(x @ wv)
    assert np.array_equal(res["out"][0], np.repeat(v_new[0][None], heads, axis=0))
    assert np.array_equal(res["v_cache"][1][2], codecs.bf16_encode(v_new[1]))
    assert np.array_equal(res["v_cache"][1][3], vc[1][3])  # row past the length untouched


# ----------------------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# ----------------------------------------------------------------------------------------


def _ln3_pin(attn_seq):
    d = 256
    q = np.zeros((1, d))
    q[0, 0] = 16.0
    k = np.zeros((2, d))
    k[0, 0] = math.log(3.0)
    v = np.stack([np.full(d, 1.0), np.full(d, 5.0)])
    return np.allclose(attn_seq(q, k, v), 0.75 * v[0] + 0.25 * v[1], rtol=0, atol=1e-12)


def test_planted_wrong_scale_is_caught():
    assert _ln3_pin(mfa.decode_attn_seq)
    assert not _ln3_pin(lambda q, k, v: mfa.decode_attn_seq(q, k, v, scale=1 / math.sqrt(255)))


def test_planted_transposed_value_product_is_caught():
    def wrong(q, k, v):  # weights applied to the wrong cache rows (reversed order of v)
        return mfa.attention_weights(q, k) @ v[::-1]
    assert not _ln3_pin(wrong)


def test_planted_eps_outside_sqrt_is_caught():
    c = np.random.default_rng(1).standard_normal((3, 2048)) * 1e-3
    m = np.mean(c * c, axis=-1)
    eps = 1e-6

    def wrong(c, g, e):
        return c / (np.sqrt(np.mean(c * c, axis=-1, keepdims=True)) + e) * g
    good = mfa.rms_norm(c, np.ones(2048), eps)
    bad = wrong(c, np.ones(2048), eps)
    assert np.allclose(np.mean(good ** 2, -1), m / (m + eps), rtol=1e-12)
    assert not np.allclose(np.mean(bad ** 2, -1), m / (m + eps), rtol=1e-9)


def test_planted_off_by_one_append_row_is_caught():
    rng = np.random.default_rng(21)
    kc = [rng.integers(0, 9, (4, 3)).astype(np.uint16)]
    new = np.full((1, 3), 77, np.uint16)
    k2, _ = mfa.kv_append(kc, kc, [2], new, new)
    assert np.array_equal(k2[0][2], new[0]) and np.array_equal(k2[0][3], kc[0][3])
    k_bad, _ = mfa.kv_append(kc, kc, [3], new, new)
    assert not np.array_equal(k_bad[0][2], new[0])


# ----------------------------------------------------------------------------------------
# output projection and the stack of layers (the attention side of a decode step)
# ----------------------------------------------------------------------------------------


@pytest.mark.parametrize("bsz,heads,hd,dout", [(1, 2, 3, 5), (3, 4, 4, 7)])
def test_o_proj_exact_on_small_integers(bsz, heads, hd, dout):
    rng = np.random.default_rng(heads * hd + dout)
    out = rng.integers(-3, 4, (bsz, heads, hd))
    w = rng.integers(-2, 3, (heads * hd, dout))
    flat = out.reshape(bsz, heads * hd).tolist()
    want = np.array(_int_matmul(flat, w.tolist()), dtype=np.float64)
    assert np.array_equal(mfa.o_proj(out, w), want)
    # the flat [B, H * d] form is the same call
    assert np.array_equal(mfa.o_proj(np.array(flat), w), want)


def test_o_proj_one_hot_copies_the_chosen_head_slot():
    # W_o routes (head h, dim j) = input column h * d + j to output column n
    heads, hd, dout = 4, 5, 9
    rng = np.random.default_rng(7)
    for _ in range(10):
        h, j, n = rng.integers(heads), rng.integers(hd), rng.integers(dout)
        w = np.zeros((heads * hd, dout))
        w[h * hd + j, n] = 1.0
        out = rng.standard_normal((3, heads, hd))
        y = mfa.o_proj(out, w)
        expect = np.zeros((3, dout))
        expect[:, n] = out[:, h, j]
        assert np.array_equal(y, expect)


def _tiny_layer(rng, dim, rank, heads, hd, lens):
    lay = dict(
        w_qdown=rng.standard_normal((dim, rank)) / math.sqrt(dim),
        gamma=rng.uniform(0.5, 1.5, rank),
        w_qup=rng.standard_normal((rank, heads * hd)) / math.sqrt(rank),
        w_k=rng.standard_normal((dim, hd)) / math.sqrt(dim),
        w_v=rng.standard_normal((dim, hd)) / math.sqrt(dim),
        w_o=rng.standard_normal((heads * hd, dim)) / math.sqrt(heads * hd))
    ck = [codecs.bf16_round(rng.standard_normal((n, hd))) for n in lens]
    cv = [codecs.bf16_round(rng.standard_normal((n, hd))) for n in lens]
    lay["k_rows"], lay["v_rows"] = ck, cv
    lay["k_cache"] = [codecs.bf16_encode(t) for t in ck]
    lay["v_cache"] = [codecs.bf16_encode(t) for t in cv]
    return lay


def test_attention_side_step_matches_brute_force_chain():
    """Two layers: layer 1's input must be layer 0's projected output, each layer's output
    projection a plain sum, and the whole chain equal to pure-Python loops."""
    rng = np.random.default_rng(11)
    dim, rank, heads, hd, lens = 10, 6, 3, 4, [3, 1, 5]
    eps, scale = 1e-6, 1.0 / math.sqrt(hd)
    layers = [_tiny_layer(rng, dim, rank, heads, hd, lens) for _ in range(2)]
    x = rng.standard_normal((len(lens), dim))
    res, y_last = mfa.attention_side_step(x, layers, lens, eps=eps, scale=scale,
                                          n_heads=heads, emulate=False)
    h = x.tolist()
    for lay, r in zip(layers, res):
        # the cache rounds the appended row to bf16; give brute force the same rows
        k_new, v_new = mfa.kv_project(np.array(h), lay["w_k"], lay["w_v"])
        ck2 = [np.vstack([lay["k_rows"][b][:lens[b] - 1], codecs.bf16_round(k_new[b])[None]])
               for b in range(len(lens))]
        cv2 = [np.vstack([lay["v_rows"][b][:lens[b] - 1], codecs.bf16_round(v_new[b])[None]])
               for b in range(len(lens))]
        out = _brute_layer(h, lay["w_qdown"].tolist(), lay["gamma"].tolist(),
                           lay["w_qup"].tolist(), lay["w_k"].tolist(), lay["w_v"].tolist(),
                           [t.tolist() for t in ck2], [t.tolist() for t in cv2], lens, heads,
                           eps, scale)
        flat = [[v for head in seq for v in head] for seq in out]
        wo = lay["w_o"].tolist()
        y = [[math.fsum(f[i] * wo[i][n] for i in range(len(f))) for n in range(dim)]
             for f in flat]
        assert np.allclose(r["out"], out, rtol=1e-12, atol=1e-13)
        assert np.allclose(r["y"], y, rtol=1e-12, atol=1e-13)
        h = y
    assert np.allclose(y_last, h, rtol=1e-12, atol=1e-13)


def test_planted_o_proj_skipped_in_the_chain_is_caught():
    # handing the attention output on without W_o changes the next layer's input
    rng = np.random.default_rng(5)
    dim, rank, heads, hd, lens = 12, 6, 3, 4, [2, 4]
    layers = [_tiny_layer(rng, dim, rank, heads, hd, lens) for _ in range(2)]
    x = rng.standard_normal((len(lens), dim))
    res, _ = mfa.attention_side_step(x, layers, lens, scale=0.5, n_heads=heads, emulate=False)
    wrong = res[0]["out"].reshape(len(lens), -1)  # heads * hd == dim: shapes would fit
    assert not np.allclose(wrong, res[0]["y"], rtol=1e-3, atol=1e-6)


# ----------------------------------------------------------------------------------------
# paged caches: the page-table layout
# ----------------------------------------------------------------------------------------


@pytest.mark.parametrize("page_size,lens", [(4, [1, 4, 9, 13]), (8, [7, 8, 17])])
def test_kv_gather_paged_reassembles_a_shuffled_cache(page_size, lens):
    rng = np.random.default_rng(page_size)
    d = 3
    seqs = [rng.integers(0, 1 << 16, (n, d)).astype(np.uint16) for n in lens]
    need = [-(-n // page_size) for n in lens]
    total = sum(need) + 3  # spare pages that no sequence uses
    order = rng.permutation(total)
    pool = np.full((total, page_size, d), 0xFFFF, dtype=np.uint16)  # poison everywhere
    tables, at = [], 0
    for s, n_pages in zip(seqs, need):
        ids = order[at:at + n_pages]
        at += n_pages
        for p, pid in enumerate(ids):
            chunk = s[p * page_size:(p + 1) * page_size]
            pool[pid][:len(chunk)] = chunk
        tables.append(ids)
    for s, ids, n in zip(seqs, tables, lens):
        assert np.array_equal(mfa.kv_gather_paged(pool, ids, n, page_size), s)
    # the page list alone decides where rows come from
    swapped = tables[2][::-1]
    if len(swapped) > 1:
        assert not np.array_equal(mfa.kv_gather_paged(pool, swapped, lens[2], page_size),
                                  seqs[2])


# ----------------------------------------------------------------------------------------
# block-FP8 weights
# ----------------------------------------------------------------------------------------


def test_w8_dequantize_places_each_block_scale():
    # power-of-two scales make every product exact: the result must be code * scale of the
    # element's own block, transposed to [in, out]
    rng = np.random.default_rng(3)
    out_dim, in_dim, blk = 10, 7, 4  # ragged last blocks in both directions
    codes = rng.integers(0, 256, (out_dim, in_dim)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x11  # no NaN codes
    scales = np.ldexp(1.0, rng.integers(-6, 6, (3, 2))).astype(np.float32)
    w = mfa.w8_dequantize(codes, scales, block=blk)
    assert w.shape == (in_dim, out_dim)
    for o in range(out_dim):
        for i in range(in_dim):
            want = codecs.e4m3_decode(codes[o, i]) * float(scales[o // blk, i // blk])
            assert w[i, o] == want


def test_a8_quantize_exact_cases():
    # max 448 * 2**-3 -> scale 2**-3 exactly; every value a multiple of the e4m3 grid
    a = np.zeros((2, 256))
    a[0, :128] = np.linspace(-56, 56, 128)
    a[0, 5] = 56.0  # the max
    a[1, 128:] = 0.0  # an all-zero group
    a[1, :128] = 3.0
    codes, scales = mfa.a8_quantize(a)
    assert scales.dtype == np.float32 and scales.shape == (2, 2)
    assert scales[0, 0] == np.float32(56.0 / 448.0) == 0.125
    assert scales[1, 1] == 1.0 and (codes[1, 128:] == 0).all()
    assert codecs.e4m3_decode(codes[0, 5]) == 448.0  # the max codes to 448
    assert codecs.e4m3_decode(codes[1, 0]) == 448.0  # 3 / (3 / 448)
    back = mfa.a8_dequantize(codes, scales)
    assert np.allclose(back[0, :128], a[0, :128], rtol=2 ** -4, atol=0)
    assert back[0, 5] == 56.0


def test_a8_quantize_brute_force():
    rng = np.random.default_rng(8)
    a = codecs.bf16_round(rng.standard_normal((3, 300)) * rng.uniform(0.01, 10, (3, 1)))
    codes, scales = mfa.a8_quantize(a)
    for r in range(3):
        for g in range(3):
            blk = a[r, 128 * g:128 * (g + 1)]
            amax = max(abs(float(v)) for v in blk)
            sc = _f32_rne(_f32_rne(amax) / 448.0)
            assert scales[r, g] == sc
            for j, v in enumerate(blk):
                q = _f32_rne(float(v) / sc)  # float32 quotient
                assert codes[r, 128 * g + j] == codecs.e4m3_encode(q)


def test_fp8_project_is_the_sum_of_real_products():
    rng = np.random.default_rng(9)
    x = codecs.bf16_round(rng.standard_normal((2, 256)))
    w = codecs.bf16_round(rng.standard_normal((256, 130)) * 0.05)  # [in, out]
    wc = codecs.e4m3_encode(w.T / 0.01)
    ws = np.full((2, 2), 0.01, np.float32)
    xc, xs = mfa.a8_quantize(x)
    want = np.zeros((2, 130))
    for b in range(2):
        for o in range(130):
            want[b, o] = math.fsum(float(codecs.e4m3_decode(xc[b, k])) * float(xs[b, k // 128])
                                   * float(codecs.e4m3_decode(wc[o, k])) * float(ws[o // 128, k // 128])
                                   for k in range(256))
    assert np.allclose(mfa.fp8_project(x, wc, ws), want, rtol=1e-12, atol=1e-12)


def _f32_rne(x):
    import struct
    return struct.unpack("<f", struct.pack("<f", x))[0]


# ----------------------------------------------------------------------------------------
# the whole FP8 query chain (step3-fp8 model card: block-fp8 checkpoints; bud-325 "Key
# claims": the model runs in FP8), brute force at tiny sizes
# ----------------------------------------------------------------------------------------


def _brute_quantize_row(row):
    """One activation row in groups of 128: (codes, scales) by the reading's rule, written
    out element by element (float32 scale and quotient, e4m3 nearest-even saturating)."""
    codes, scales = [], []
    for g0 in range(0, len(row), 128):
        grp = [float(v) for v in row[g0:g0 + 128]]
        amax = max(abs(v) for v in grp)
        sc = _f32_rne(_f32_rne(amax) / 448.0) if amax > 0 else 1.0
        scales.append(sc)
        codes.extend(int(codecs.e4m3_encode(_f32_rne(v / sc))) for v in grp)
    return codes, scales


def _brute_fp8_dot(a_codes, a_scales, w_codes, w_scales, o):
    """sum_k a_k w[o, k] over the real values code * scale, as one exact-rounded fsum."""
    return math.fsum(float(codecs.e4m3_decode(a_codes[k])) * a_scales[k // 128]
                     * float(codecs.e4m3_decode(w_codes[o, k])) * float(w_scales[o // 128, k // 128])
                     for k in range(len(a_codes)))


def _brute_query_proj_fp8(x, wq_codes, wq_scales, gamma, wu_codes, wu_scales, n_heads, eps):
    """The FP8 query path in pure Python: x quantized per group, c by exact sums, RMSNorm,
    c_hat rounded to bf16 (as stored) and only then quantized, q by exact sums, rounded to
    bf16, and q[b][h][d] taken from output column h * head_dim + d (head-major)."""
    rank = wq_codes.shape[0]
    width = wu_codes.shape[0]
    hd = width // n_heads
    c_hat_all, q_all = [], []
    for row in x:
        xc, xs = _brute_quantize_row(row)
        c = [_brute_fp8_dot(xc, xs, wq_codes, wq_scales, r) for r in range(rank)]
        inv = 1.0 / math.sqrt(math.fsum(v * v for v in c) / rank + eps)
        c_hat = [float(codecs.bf16_round(v * inv * float(gamma[j]))) for j, v in enumerate(c)]
        cc, cs = _brute_quantize_row(c_hat)
        q = [[float(codecs.bf16_round(_brute_fp8_dot(cc, cs, wu_codes, wu_scales, h * hd + d)))
              for d in range(hd)] for h in range(n_heads)]
        c_hat_all.append(c_hat)
        q_all.append(q)
    return np.array(c_hat_all), np.array(q_all)


def _fp8_chain_inputs(seed=21, bsz=2, din=256, rank=256, n_heads=3, hd=64):
    rng = np.random.default_rng(seed)
    x = codecs.bf16_round(rng.standard_normal((bsz, din)) * rng.uniform(0.2, 5.0, (bsz, 1)))
    wq = rng.standard_normal((rank, din)) / math.sqrt(din)          # [out, in]
    wu = rng.standard_normal((n_heads * hd, rank)) / math.sqrt(rank)
    # block scales of different sizes per 128 x 128 block (the output side of W_qup ends in a
    # ragged block of 64)
    wq_s = np.array([[0.004, 0.003], [0.005, 0.0035]], np.float32)
    wu_s = np.array([[0.006, 0.0045], [0.005, 0.007]], np.float32)
    wq_c = codecs.e4m3_encode(wq / np.repeat(np.repeat(wq_s, 128, 0), 128, 1)[:rank, :din])
    wu_c = codecs.e4m3_encode(wu / np.repeat(np.repeat(wu_s, 128, 0), 128, 1)[:n_heads * hd, :rank])
    gamma = codecs.bf16_round(rng.uniform(0.5, 1.5, rank))
    return x, wq_c, wq_s, gamma, wu_c, wu_s, n_heads


_BRUTE_FP8 = {}


def _brute_fp8_chain():
    """The brute force of the default chain inputs, computed once for the tests below."""
    if not _BRUTE_FP8:
        x, wq_c, wq_s, gamma, wu_c, wu_s, nh = _fp8_chain_inputs()
        _BRUTE_FP8["r"] = _brute_query_proj_fp8(x, wq_c, wq_s, gamma, wu_c, wu_s, nh,
                                                mfa.RMS_EPS)
    return _BRUTE_FP8["r"]


def test_query_proj_fp8_matches_pure_python_brute_force():
    x, wq_c, wq_s, gamma, wu_c, wu_s, nh = _fp8_chain_inputs()
    c_hat, q = mfa.query_proj_fp8(x, wq_c, wq_s, gamma, wu_c, wu_s, n_heads=nh)
    bc, bq = _brute_fp8_chain()
    assert q.shape == bq.shape == (2, 3, 64)
    # both sides round the same real numbers to bf16: equal unless a float64 sum sits within
    # 1e-16 of a rounding midpoint
    assert np.array_equal(c_hat, bc)
    assert np.array_equal(q, bq)


def test_query_proj_fp8_one_hot_routes_to_the_head_major_slot():
    # W_qup with one nonzero code per output column: column h * 64 + d reads input j(h, d),
    # so q[b, h, d] must be (the e4m3 code of c_hat[j] in its group) * scales, rounded to bf16
    x, wq_c, wq_s, gamma, _, _, nh = _fp8_chain_inputs(seed=5)
    hd, rank = 64, 256
    wu_c = np.zeros((nh * hd, rank), np.uint8)
    wu_s = np.array([[0.25, 0.5], [2.0, 1.0]], np.float32)
    one = int(codecs.e4m3_encode(1.0))
    src = {}
    for h in range(nh):
        for d in range(hd):
            j = (7 * h + 3 * d + 11) % rank
            wu_c[h * hd + d, j] = one
            src[h, d] = j
    c_hat, q = mfa.query_proj_fp8(x, wq_c, wq_s, gamma, wu_c, wu_s, n_heads=nh)
    for b in range(2):
        cc, cs = _brute_quantize_row(c_hat[b])
        for (h, d), j in src.items():
            o = h * hd + d
            want = codecs.bf16_round(float(codecs.e4m3_decode(cc[j])) * cs[j // 128]
                                     * float(wu_s[o // 128, j // 128]))
            assert q[b, h, d] == want


def test_planted_fp8_quantize_before_bf16_rounding_is_caught():
    # a chain that quantizes the float64 c_hat (before its storage rounding to bf16) differs
    # from the stated order; the brute-force pin must reject it
    x, wq_c, wq_s, gamma, wu_c, wu_s, nh = _fp8_chain_inputs()

    def wrong_order(x, wq_c, wq_s, gamma, wu_c, wu_s, n_heads):
        c_hat = mfa.rms_norm(mfa.fp8_project(x, wq_c, wq_s), gamma)
        q = codecs.bf16_round(mfa.fp8_project(c_hat, wu_c, wu_s))
        return q.reshape(q.shape[0], n_heads, -1)

    _, bq = _brute_fp8_chain()
    assert not np.array_equal(wrong_order(x, wq_c, wq_s, gamma, wu_c, wu_s, nh), bq)


def test_planted_fp8_dim_major_reshape_is_caught():
    # q taken dim-major ([b, head_dim, heads] then transposed) instead of head-major
    x, wq_c, wq_s, gamma, wu_c, wu_s, nh = _fp8_chain_inputs()
    _, q = mfa.query_proj_fp8(x, wq_c, wq_s, gamma, wu_c, wu_s, n_heads=nh)
    flat = q.reshape(q.shape[0], -1)
    wrong = flat.reshape(q.shape[0], -1, nh).transpose(0, 2, 1)
    _, bq = _brute_fp8_chain()
    assert np.array_equal(q, bq) and not np.array_equal(wrong, bq)
