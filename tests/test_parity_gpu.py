"""GPU parity of the CUDA path (called through the C ABI) against the float64 oracle on the
same seeded inputs: per op (the oracle reads the GPU-visible inputs of that op) and end to
end (the oracle's own chain), small cases spanning several tiles and ragged tails, edge
lengths, forced split-K, device-side error paths, and the five named workloads (sampled
sequences at full size)."""

import numpy as np
import pytest
import torch

from decode_attention_10_b200 import workloads as W
from oracle import codecs
from oracle import mfa as omfa

from mfa_util import (GpuStep, assert_close, bf16_np, codes_np, max_abs, oracle_dtype,
                      oracle_weights, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from decode_attention_10_b200 import build, mfa
    build.build()
    mfa.load()


def _q_close(q_gpu, q_ref):
    # q is stored as bf16 on both sides; allow two bf16 ulps of the reference value plus a
    # small absolute slack for values whose normalized input rounded differently
    ulp = np.ldexp(1.0, np.frexp(np.abs(q_ref))[1] - 8)
    bad = np.abs(q_gpu - q_ref) > 2 * ulp + 1e-3
    assert not bad.any(), f"{bad.sum()} q elements off, max {max_abs(q_gpu, q_ref):.3e}"
    assert rel_l2(q_gpu, q_ref) <= 1e-3


def _check_layer(inp: W.Inputs, sample=None, e2e=True):
    step = GpuStep(inp)
    k_before = [codes_np(t) for t in step.k]
    v_before = [codes_np(t) for t in step.v]
    q_gpu, out_gpu = step.layer()
    torch.cuda.synchronize()
    from decode_attention_10_b200 import mfa
    assert mfa.get_error(step.ws) == 0
    bsz = inp.batch
    seqs = list(range(bsz)) if sample is None else sample
    lens = inp.seq_lens.tolist()
    od = oracle_dtype(inp.kv_dtype)
    ow = oracle_weights(inp)
    xs = ow["x"][seqs]
    # query path
    _, q_ref = omfa.query_proj(xs, ow["w_qdown"], ow["gamma"], ow["w_qup"])
    q_np = bf16_np(q_gpu)[seqs]
    _q_close(q_np, q_ref)
    # appended rows: one code apart at most (fp32 vs float64 rounding decision); every
    # other byte of the cache unchanged
    k_new, v_new = omfa.kv_project(xs, ow["w_k"], ow["w_v"])
    k_codes = omfa.kv_store(k_new, od, inp.k_scale)
    v_codes = omfa.kv_store(v_new, od, inp.v_scale)
    k_after = {b: codes_np(step.k[b]) for b in seqs}
    v_after = {b: codes_np(step.v[b]) for b in seqs}
    for i, b in enumerate(seqs):
        row = lens[b] - 1
        for after, before, want in ((k_after[b], k_before[b], k_codes[i]),
                                    (v_after[b], v_before[b], v_codes[i])):
            rest = np.ones(after.shape[0], bool)
            rest[row] = False
            assert np.array_equal(after[rest], before[rest]), f"seq {b}: other rows changed"
            got = after[row].astype(np.int64)
            diff = np.abs(got - want.astype(np.int64))
            assert diff.max() <= 1, f"seq {b}: appended row differs by {diff.max()} codes"
            assert (diff != 0).mean() < 0.01
    # attention, per op: the oracle reads the GPU's q and the GPU's cache after the append
    out_np = bf16_np(out_gpu)[seqs]
    k_list = [k_after[b] for b in seqs]
    v_list = [v_after[b] for b in seqs]
    ref = omfa.decode_attn(q_np, k_list, v_list, [lens[b] for b in seqs], od, inp.k_scale,
                           inp.v_scale)
    res = assert_close(out_np, ref, inp.kv_dtype, "attention (per op)")
    if e2e:
        # end to end: the oracle's own chain from x, weights and the original cache
        kc = [k_before[b] for b in seqs]
        vc = [v_before[b] for b in seqs]
        full = omfa.decode_layer(xs, ow["w_qdown"], ow["gamma"], ow["w_qup"], ow["w_k"],
                                 ow["w_v"], kc, vc, [lens[b] for b in seqs], od, inp.k_scale,
                                 inp.v_scale)
        assert_close(out_np, full["out"], inp.kv_dtype, "layer (end to end)")
    return res


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_layer_small_ragged(kv_dtype):
    # lengths span one and several 128-position tiles with ragged tails
    inp = W.generate([1, 130, 300, 129, 128, 2], kv_dtype, seed=11)
    _check_layer(inp)


def test_layer_batch_over_256_rows():
    # the weight GEMMs take token rows in slices of 256 (a second grid slice from row 256):
    # rows on both sides of the seam
    g = np.random.default_rng(41)
    lens = [int(x) for x in g.integers(1, 300, size=300)]
    inp = W.generate(lens, W.KV_BF16, seed=41, contiguous=False)
    _check_layer(inp, sample=[0, 1, 128, 255, 256, 257, 299], e2e=True)


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_layer_max_batch(kv_dtype):
    # MFA_MAX_BATCH sequences through the whole step: the plan's arrays full, several work
    # items per attention CTA, short sequences split across CTA boundaries
    from decode_attention_10_b200 import mfa
    g = np.random.default_rng(42)
    lens = [int(x) for x in g.integers(1, 400, size=mfa.MAX_BATCH)]
    inp = W.generate(lens, kv_dtype, seed=42, contiguous=False)
    _check_layer(inp, sample=[0, 1, 147, 148, 511, 512, 1022, 1023], e2e=True)


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_attention_max_batch_every_sequence(kv_dtype):
    # every one of MFA_MAX_BATCH outputs against the oracle (attention alone)
    from decode_attention_10_b200 import mfa
    g = np.random.default_rng(43)
    lens = [int(x) for x in g.integers(1, 400, size=mfa.MAX_BATCH)]
    out, ref, _ = _attn_case(lens, kv_dtype, seed=43)
    assert_close(out, ref, kv_dtype, "max batch")


def test_layer_per_sequence_buffers_with_spare_capacity():
    lens = [77, 513, 1]
    caps = [100, 600, 9]
    inp = W.generate(lens, W.KV_BF16, seed=12, contiguous=False, capacity=caps)
    _check_layer(inp)


def _attn_case(lens, kv_dtype, seed, caps=None, nan_tail=False, q_scale=1.0, ws=None):
    from decode_attention_10_b200 import mfa
    inp = W.generate(lens, kv_dtype, seed=seed, contiguous=False, capacity=caps)
    g = torch.Generator().manual_seed(seed + 7)
    q = (torch.randn(len(lens), 64, 256, generator=g) * q_scale).to(torch.bfloat16)
    k = [t.clone() for t in inp.k_cache]
    v = [t.clone() for t in inp.v_cache]
    if nan_tail:  # rows past the length hold NaN patterns: they must not leak into out
        for kt, vt, n in zip(k, v, lens):
            kt.view(torch.uint8)[n:] = 0x7F if kv_dtype == W.KV_FP8 else 0xFF
            vt.view(torch.uint8)[n:] = 0x7F if kv_dtype == W.KV_FP8 else 0xFF
    kd = [t.cuda() for t in k]
    vd = [t.cuda() for t in v]
    cache = mfa.KVCache(kd, vd, inp.k_scale, inp.v_scale)
    out = mfa.decode_attn(q.cuda(), cache, inp.seq_lens.cuda(), ws=ws)
    torch.cuda.synchronize()
    ref = omfa.decode_attn(bf16_np(q), [codes_np(t) for t in k], [codes_np(t) for t in v],
                           lens, oracle_dtype(kv_dtype), inp.k_scale, inp.v_scale)
    return bf16_np(out), ref, cache


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_attention_edge_lengths(kv_dtype):
    lens = [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 1000]
    out, ref, _ = _attn_case(lens, kv_dtype, seed=21)
    assert_close(out, ref, kv_dtype, "edge lengths")
    # L = 1: every head's output is the single cached V row (exact for bf16 caches; for FP8
    # the value code * scale is rounded to bf16 once more, within one bf16 ulp)
    want = np.repeat(ref[0][:1], 64, axis=0)
    if kv_dtype == W.KV_BF16:
        assert np.array_equal(out[0], want)
    else:
        ulp = np.ldexp(1.0, np.frexp(np.abs(want))[1] - 8)
        assert (np.abs(out[0] - want) <= ulp).all()


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_attention_rows_past_length_are_ignored(kv_dtype):
    lens = [5, 130, 300]
    caps = [64, 256, 512]
    out, ref, _ = _attn_case(lens, kv_dtype, seed=22, caps=caps, nan_tail=True)
    assert np.isfinite(out).all()
    assert_close(out, ref, kv_dtype, "NaN past length")


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_attention_long_sequence_split_over_many_ctas(kv_dtype):
    # one 40,000-position sequence spans ~313 tiles, more than one per SM: it is split over
    # every CTA, and the merge takes the path for more than 8 splits
    out, ref, _ = _attn_case([40000], kv_dtype, seed=23)
    assert_close(out, ref, kv_dtype, "long single sequence")
    out, ref, _ = _attn_case([65536, 3, 20000], kv_dtype, seed=24)
    assert_close(out, ref, kv_dtype, "mixed long")


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
@pytest.mark.parametrize("shape", ["few_sequences", "large_batch"])
def test_attention_every_combine_path(kv_dtype, shape):
    # The combine merges a split sequence in one of four ways: batches under 64 sequences with
    # 2 heads per thread, in one round trip up to 6 splits and through shared-memory weights
    # beyond; batches of 64 and more with 4 heads per thread, one round trip up to 3 splits.
    # Each case below reaches both ways of its shape (checked on the device's own plan).
    from decode_attention_10_b200 import mfa
    if shape == "few_sequences":
        lens = [20000, 6000, 1500, 700, 520, 129, 64, 3]
        one_pass_max = 6
    else:
        rng = np.random.default_rng(71)
        lens = [30000, 8000, 2000] + rng.integers(250, 700, 45).tolist() + [1, 2] * 8
        one_pass_max = 3
    out, ref, cache = _attn_case(lens, kv_dtype, seed=70 if shape == "few_sequences" else 71)
    _, _, items = mfa.split_plan(cache, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                 torch.cuda.get_device_properties(0).multi_processor_count)
    ns = {int(b): int(n) for b, n in zip(items[:, 1], items[:, 5])}
    splits = set(ns.values())
    assert any(2 <= n <= one_pass_max for n in splits), splits  # one round trip
    assert any(n > one_pass_max for n in splits), splits        # two phases
    assert 1 in splits                                          # finished in place
    assert_close(out, ref, kv_dtype, f"combine paths ({shape})")


def test_attention_one_workspace_across_differently_split_calls():
    # One workspace across calls whose sequences split differently (2 to 148 CTAs per
    # sequence, sequences finished by one CTA alone, lengths of 1 and 5). Each call rewrites
    # the per-sequence split information and the partial slots in the workspace; nothing an
    # earlier call left there may reach a later call's merge.
    from decode_attention_10_b200 import mfa
    ws = mfa.Workspace(16)
    cases = [[9000, 300, 20000], [40000], [700] * 16, [5, 4096, 1, 65, 12000],
             [9000, 300, 20000]]
    outs = []
    for i, lens in enumerate(cases):
        out, ref, _ = _attn_case(lens, W.KV_BF16, seed=60 + (i % 4), ws=ws)
        assert mfa.get_error(ws) == 0
        assert_close(out, ref, W.KV_BF16, f"call {i} on one workspace")
        outs.append(out)
    # the combine adds the splits in a fixed order: the same call gives the same bits
    assert np.array_equal(outs[0], outs[4])


def test_attention_sharp_softmax():
    # large scores: the running max changes often and by a lot
    out, ref, _ = _attn_case([3000, 700], W.KV_BF16, seed=25, q_scale=12.0)
    assert_close(out, ref, W.KV_BF16, "sharp softmax")


def test_attention_split_invariance():
    # the same sequence alone, and batched with others (so it is split differently and its
    # tiles start at different positions), gives the same output up to the rounding of the
    # path: both runs round P and out to bf16, each about 1.5e-3 relative
    from decode_attention_10_b200 import mfa
    inp = W.generate([9000, 300, 20000], W.KV_BF16, seed=26, contiguous=False)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(3, 64, 256, generator=g).to(torch.bfloat16).cuda()
    kd = [t.cuda() for t in inp.k_cache]
    vd = [t.cuda() for t in inp.v_cache]
    full = mfa.decode_attn(q, mfa.KVCache(kd, vd), inp.seq_lens.cuda())
    alone = mfa.decode_attn(q[:1].contiguous(), mfa.KVCache(kd[:1], vd[:1]),
                            inp.seq_lens[:1].cuda())
    a, b = bf16_np(full[:1]), bf16_np(alone)
    assert rel_l2(a, b) < 5e-3 and max_abs(a, b) < 2e-3


def test_device_errors_zero_fill_and_report():
    from decode_attention_10_b200 import mfa
    inp = W.generate([50, 60, 70], W.KV_BF16, seed=27, contiguous=False)
    kd = [t.cuda() for t in inp.k_cache]
    vd = [t.cuda() for t in inp.v_cache]
    cache = mfa.KVCache(kd, vd)
    ws = mfa.Workspace(3)
    g = torch.Generator().manual_seed(3)
    q = torch.randn(3, 64, 256, generator=g).to(torch.bfloat16).cuda()
    lens = torch.tensor([50, 61, 70], dtype=torch.int32).cuda()  # 61 > capacity 60
    out = mfa.decode_attn(q, cache, lens, ws=ws)
    assert mfa.get_error(ws) == 3  # MFA_ERR_CAPACITY
    assert mfa.get_error(ws) == 0  # cleared
    assert (out[1].float() == 0).all()
    ref = omfa.decode_attn(bf16_np(q), [codes_np(t) for t in inp.k_cache],
                           [codes_np(t) for t in inp.v_cache], [50, 60, 70])
    o = bf16_np(out)
    assert_close(o[[0, 2]], ref[[0, 2]], what="healthy sequences")
    lens = torch.tensor([50, 0, 70], dtype=torch.int32).cuda()
    out = mfa.decode_attn(q, cache, lens, ws=ws)
    assert mfa.get_error(ws) == 6  # MFA_ERR_EMPTY
    assert (out[1].float() == 0).all()
    # append at a row past the capacity: nothing written, flagged
    before = [codes_np(t) for t in kd]
    pos = torch.tensor([0, 60, 3], dtype=torch.int32).cuda()
    mfa.kv_append(inp.x.cuda(), inp.w_k.cuda(), inp.w_v.cuda(), cache, pos, ws=ws)
    assert mfa.get_error(ws) == 3
    after = [codes_np(t) for t in kd]
    assert np.array_equal(after[1], before[1])


def test_bounded_wait_expires_reports_timeout_and_context_survives():
    """Failure detection without a fault: a kernel waits, through the library's bounded
    mbarrier wait, on a barrier that nothing completes. The wait must give up after its
    limit, the call must report MFA_ERR_TIMEOUT, and the same context and workspace must
    still compute correct attention afterwards."""
    import time
    from decode_attention_10_b200 import mfa
    ws = mfa.Workspace(4)
    assert mfa.get_error(ws) == 0
    t0 = time.perf_counter()
    mfa.wait_selftest(ws, limit_us=2000)
    assert mfa.get_error(ws) == 7  # MFA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0  # ended by its own bound, far below any watchdog
    assert mfa.get_error(ws) == 0  # cleared
    with pytest.raises(mfa.MfaError):
        mfa.wait_selftest(ws, limit_us=0)  # out of range: rejected on the host
    # the context is intact: a normal attention call on the same workspace is exact
    inp = W.generate([1, 130, 300, 40], W.KV_BF16, seed=31, contiguous=False)
    cache = mfa.KVCache([t.cuda() for t in inp.k_cache], [t.cuda() for t in inp.v_cache])
    g = torch.Generator().manual_seed(5)
    q = torch.randn(4, 64, 256, generator=g).to(torch.bfloat16)
    out = mfa.decode_attn(q.cuda(), cache, inp.seq_lens.cuda(), ws=ws)
    assert mfa.get_error(ws) == 0
    ref = omfa.decode_attn(bf16_np(q), [codes_np(t) for t in inp.k_cache],
                           [codes_np(t) for t in inp.v_cache], inp.seq_lens.tolist())
    assert_close(bf16_np(out), ref, what="attention after an expired wait")


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_kv_append_bit_exact(kv_dtype):
    """One-hot W makes k and v exact copies of chosen elements of x; with values on the
    cache grid (and a power-of-two FP8 scale) the stored bytes are known exactly."""
    from decode_attention_10_b200 import mfa
    bsz, caps = 5, [3, 8, 1, 130, 64]
    rng = np.random.default_rng(3)
    fp8 = kv_dtype == W.KV_FP8
    k_scale, v_scale = (0.5, 0.25) if fp8 else (1.0, 1.0)
    if fp8:
        # nonzero grid values: a dot product of -0 with +0 terms is +0, not -0
        grid = codecs.e4m3_decode(np.arange(1, 0x7F))
        xv = rng.choice(grid, (bsz, 7168)) * rng.choice([-1.0, 1.0], (bsz, 7168)) * 0.25
    else:
        xv = codecs.bf16_round(rng.standard_normal((bsz, 7168)))
    x = torch.from_numpy(codecs.bf16_encode(xv).view(np.int16)).view(torch.bfloat16)
    pk, pv = rng.permutation(7168)[:256], rng.permutation(7168)[:256]
    wk = torch.zeros(7168, 256)
    wv = torch.zeros(7168, 256)
    wk[pk, np.arange(256)] = 1.0
    wv[pv, np.arange(256)] = 2.0
    dt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    k = [torch.zeros(c, 256).to(dt).cuda() for c in caps]
    v = [torch.zeros(c, 256).to(dt).cuda() for c in caps]
    for t in k + v:
        t.view(torch.uint8).fill_(0x5A)  # canary bytes
    cache = mfa.KVCache(k, v, k_scale, v_scale)
    pos = [2, 7, 0, 129, 31]
    mfa.kv_append(x.cuda(), wk.to(torch.bfloat16).cuda(), wv.to(torch.bfloat16).cuda(), cache,
                  torch.tensor(pos, dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    od = oracle_dtype(kv_dtype)
    kexp = omfa.kv_store(xv[:, pk], od, k_scale)
    vexp = omfa.kv_store(2.0 * xv[:, pv], od, v_scale)
    for b in range(bsz):
        kb, vb = codes_np(k[b]), codes_np(v[b])
        assert np.array_equal(kb[pos[b]], kexp[b]) and np.array_equal(vb[pos[b]], vexp[b])
        rest = np.ones(caps[b], bool)
        rest[pos[b]] = False
        canary = 0x5A5A if not fp8 else 0x5A
        assert (kb[rest] == canary).all() and (vb[rest] == canary).all()


def test_query_proj_matches_oracle():
    from decode_attention_10_b200 import mfa
    inp = W.generate([1] * 37, W.KV_BF16, seed=31)  # a batch that is not a tile multiple
    q = mfa.query_proj(inp.x.cuda(), inp.w_qdown.cuda(), inp.gamma.cuda(), inp.w_qup.cuda())
    torch.cuda.synchronize()
    ow = oracle_weights(inp)
    _, q_ref = omfa.query_proj(ow["x"], ow["w_qdown"], ow["gamma"], ow["w_qup"])
    _q_close(bf16_np(q), q_ref)


def test_query_proj_nonunit_gamma_and_scaled_input():
    from decode_attention_10_b200 import mfa
    inp = W.generate([1] * 3, W.KV_BF16, seed=32, x_scale=1e-3)
    g = torch.Generator().manual_seed(1)
    gamma = (0.5 + torch.rand(2048, generator=g)).to(torch.bfloat16)
    q = mfa.query_proj(inp.x.cuda(), inp.w_qdown.cuda(), gamma.cuda(), inp.w_qup.cuda())
    torch.cuda.synchronize()
    ow = oracle_weights(inp)
    _, q_ref = omfa.query_proj(ow["x"], ow["w_qdown"], bf16_np(gamma), ow["w_qup"])
    _q_close(bf16_np(q), q_ref)


@pytest.mark.slow
@pytest.mark.parametrize("index", [0, 1, 2, 3, 4])
def test_named_workload_sampled(index):
    w = W.workload(index)
    inp = W.generate_workload(w)
    b = inp.batch
    sample = sorted(set([0, b // 3, b // 2, b - 1]))
    _check_layer(inp, sample=sample, e2e=True)


# ----------------------------------------------------------------------------------------
# output projection, and the attention side of a step through a stack of layers
# ----------------------------------------------------------------------------------------


def _y_close(y_gpu, y_ref):
    # y is stored as bf16, so the float64 reference is rounded to bf16 as the oracle's
    # emulation does for stored tensors; then two bf16 ulps plus a small absolute slack
    y_ref = codecs.bf16_round(y_ref)
    ulp = np.ldexp(1.0, np.frexp(np.abs(y_ref))[1] - 8)
    bad = np.abs(y_gpu - y_ref) > 2 * ulp + 1e-4
    assert not bad.any(), f"{bad.sum()} y elements off, max {max_abs(y_gpu, y_ref):.3e}"
    assert rel_l2(y_gpu, y_ref) <= 1e-3


@pytest.mark.parametrize("bsz", [1, 32, 300])
def test_o_proj_matches_oracle(bsz):
    from decode_attention_10_b200 import mfa
    g = torch.Generator().manual_seed(40 + bsz)
    out = (torch.randn(bsz, 64, 256, generator=g) * 0.05).to(torch.bfloat16)
    w_o = W.generate_w_o(41)
    y = mfa.o_proj(out.cuda(), w_o.cuda())
    torch.cuda.synchronize()
    # every 7th output column: all 56 tiles of 128 features, both split-K halves
    cols = np.arange(0, 7168, 7)
    ref = omfa.o_proj(bf16_np(out), bf16_np(w_o[:, cols]))
    _y_close(bf16_np(y)[:, cols], ref)


def test_o_proj_bit_exact_on_small_integers():
    # integer inputs: every fp32 partial sum is exact (|y| <= 16384 * 6 < 2**24), so the
    # split-K order cannot matter and y must equal bf16(exact) bit for bit
    from decode_attention_10_b200 import mfa
    g = torch.Generator().manual_seed(43)
    out = torch.randint(-3, 4, (40, 64, 256), generator=g).to(torch.bfloat16)
    w_o = torch.randint(-2, 3, (16384, 7168), generator=g).to(torch.bfloat16)
    y = mfa.o_proj(out.cuda(), w_o.cuda())
    torch.cuda.synchronize()
    cols = np.arange(3, 7168, 11)
    exact = omfa.o_proj(bf16_np(out), bf16_np(w_o[:, cols]))
    got = codes_np(y)[:, cols]
    assert np.array_equal(got, codecs.bf16_encode(exact))


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_attention_side_two_layers(kv_dtype):
    """Two layers chained on one stream as a serving loop runs them: layer 1's hidden input
    is layer 0's projected output. Per layer the oracle reads the GPU's own inputs of that
    layer; end to end it runs its own chain from x and the original caches."""
    from decode_attention_10_b200 import mfa
    lens = [1, 130, 300]
    inps = [W.generate(lens, kv_dtype, seed=60 + l) for l in range(2)]
    w_os = [W.generate_w_o(70 + l) for l in range(2)]
    steps = [GpuStep(inp) for inp in inps]
    k_before = [[codes_np(t) for t in st.k] for st in steps]
    v_before = [[codes_np(t) for t in st.v] for st in steps]
    x = steps[0].x
    xs, outs, ys = [], [], []
    for st, w_o in zip(steps, w_os):
        _, out = mfa.decode_layer(x, st.w_qdown, st.gamma, st.w_qup, st.w_k, st.w_v, st.cache,
                                  st.seq_lens, ws=st.ws)
        y = mfa.o_proj(out, w_o.cuda(), ws=st.ws)
        xs.append(x)
        outs.append(out)
        ys.append(y)
        x = y
    torch.cuda.synchronize()
    assert all(mfa.get_error(st.ws) == 0 for st in steps)
    od = oracle_dtype(kv_dtype)
    layers = []
    for l, (inp, st) in enumerate(zip(inps, steps)):
        ow = oracle_weights(inp)
        lay = dict(w_qdown=ow["w_qdown"], gamma=ow["gamma"], w_qup=ow["w_qup"], w_k=ow["w_k"],
                   w_v=ow["w_v"], w_o=bf16_np(w_os[l]), k_cache=k_before[l],
                   v_cache=v_before[l], k_scale=inp.k_scale, v_scale=inp.v_scale)
        layers.append(lay)
        # per layer: the GPU's own hidden input of this layer
        r = omfa.decode_layer(bf16_np(xs[l]), lay["w_qdown"], lay["gamma"], lay["w_qup"],
                              lay["w_k"], lay["w_v"], lay["k_cache"], lay["v_cache"], lens, od,
                              inp.k_scale, inp.v_scale)
        assert_close(bf16_np(outs[l]), r["out"], kv_dtype, f"layer {l} attention")
        _y_close(bf16_np(ys[l]), omfa.o_proj(bf16_np(outs[l]), lay["w_o"]))
    # end to end through both layers: two layers' worth of the per-layer tolerance
    _, y_ref = omfa.attention_side_step(oracle_weights(inps[0])["x"], layers, lens, od)
    assert rel_l2(bf16_np(ys[-1]), y_ref) <= 2 * 5e-3


# ----------------------------------------------------------------------------------------
# paged KV caches (page tables, shuffled pages, unused rows poisoned with NaN)
# ----------------------------------------------------------------------------------------


def _paged_from(inp: W.Inputs, page_size: int, seed: int, spare: int = 5):
    """The caches of ``inp`` copied into shuffled pages of K and V pools. Rows past each
    sequence's length, and unused pages, hold NaN codes. Returns (PagedKVCache, k_pool,
    v_pool, page_table (host numpy), pages per sequence)."""
    from decode_attention_10_b200 import mfa
    rng = np.random.default_rng(seed)
    lens = inp.seq_lens.tolist()
    caps = inp.meta["capacity"]
    need = [-(-c // page_size) for c in caps]
    total = sum(need) + spare
    order = rng.permutation(total)
    fp8 = inp.kv_dtype == W.KV_FP8
    nan_code = 0x7F if fp8 else 0x7FC0
    np_dtype = np.uint8 if fp8 else np.uint16
    pools = []
    table = np.zeros((len(lens), max(need)), dtype=np.int32)
    at = 0
    for b, n_pages in enumerate(need):
        table[b, :n_pages] = order[at:at + n_pages]
        at += n_pages
    for cache in (inp.k_cache, inp.v_cache):
        pool = np.full((total, page_size, 256), nan_code, dtype=np_dtype)
        for b, n in enumerate(lens):
            rows = codes_np(cache[b])[:n]
            for p in range(need[b]):
                chunk = rows[p * page_size:(p + 1) * page_size]
                pool[table[b, p], :len(chunk)] = chunk
        t = torch.from_numpy(pool.view(np.int8 if fp8 else np.int16))
        t = t.view(torch.float8_e4m3fn if fp8 else torch.bfloat16)
        pools.append(t.cuda())
    pt = torch.from_numpy(table).cuda()
    cache = mfa.PagedKVCache(pools[0], pools[1], pt, need, inp.k_scale, inp.v_scale)
    return cache, pools[0], pools[1], table, need


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
@pytest.mark.parametrize("page_size", [64, 128, 256, 512])
def test_paged_attention_matches_oracle(kv_dtype, page_size):
    from decode_attention_10_b200 import mfa
    lens = [1, 130, 300, 129, 128, 2, 777, 64]
    inp = W.generate(lens, kv_dtype, seed=80 + page_size)
    cache, k_pool, v_pool, table, need = _paged_from(inp, page_size, seed=page_size)
    g = torch.Generator().manual_seed(81)
    q = torch.randn(len(lens), 64, 256, generator=g).to(torch.bfloat16).cuda()
    seq_lens = inp.seq_lens.cuda()
    ws = mfa.Workspace(len(lens))
    out = mfa.decode_attn(q, cache, seq_lens, ws=ws)
    torch.cuda.synchronize()
    assert mfa.get_error(ws) == 0
    od = oracle_dtype(kv_dtype)
    kp, vp = codes_np(k_pool), codes_np(v_pool)
    k_rows = [omfa.kv_gather_paged(kp, table[b], n, page_size) for b, n in enumerate(lens)]
    v_rows = [omfa.kv_gather_paged(vp, table[b], n, page_size) for b, n in enumerate(lens)]
    for b, n in enumerate(lens):  # the layout itself: the pages hold the original rows
        assert np.array_equal(k_rows[b], codes_np(inp.k_cache[b])[:n])
    ref = omfa.decode_attn(bf16_np(q), k_rows, v_rows, lens, od, inp.k_scale, inp.v_scale)
    out_np = bf16_np(out)
    assert np.isfinite(out_np).all()
    assert_close(out_np, ref, kv_dtype, f"paged attention, page size {page_size}")


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_paged_layer_appends_into_the_right_page(kv_dtype):
    from decode_attention_10_b200 import mfa
    page_size = 128
    # lengths whose appended row opens a fresh page (129, 257), ends one (128), or sits
    # inside one
    lens = [129, 128, 257, 5, 400]
    inp = W.generate(lens, kv_dtype, seed=90, capacity=[c + 60 for c in lens])
    cache, k_pool, v_pool, table, need = _paged_from(inp, page_size, seed=91)
    k_before, v_before = codes_np(k_pool).copy(), codes_np(v_pool).copy()
    step = GpuStep(inp)
    q, out = mfa.decode_layer(step.x, step.w_qdown, step.gamma, step.w_qup, step.w_k, step.w_v,
                              cache, step.seq_lens, ws=step.ws)
    torch.cuda.synchronize()
    assert mfa.get_error(step.ws) == 0
    od = oracle_dtype(kv_dtype)
    ow = oracle_weights(inp)
    k_new, v_new = omfa.kv_project(ow["x"], ow["w_k"], ow["w_v"])
    k_codes = omfa.kv_store(k_new, od, inp.k_scale)
    v_codes = omfa.kv_store(v_new, od, inp.v_scale)
    kp, vp = codes_np(k_pool), codes_np(v_pool)
    for pool, before, want in ((kp, k_before, k_codes), (vp, v_before, v_codes)):
        changed = np.zeros(pool.shape[:2], bool)
        for b, n in enumerate(lens):
            page, r = table[b, (n - 1) // page_size], (n - 1) % page_size
            changed[page, r] = True
            diff = np.abs(pool[page, r].astype(np.int64) - want[b].astype(np.int64))
            assert diff.max() <= 1, f"seq {b}: appended row differs by {diff.max()} codes"
        assert np.array_equal(pool[~changed], before[~changed]), "other rows changed"
    k_rows = [omfa.kv_gather_paged(kp, table[b], n, page_size) for b, n in enumerate(lens)]
    v_rows = [omfa.kv_gather_paged(vp, table[b], n, page_size) for b, n in enumerate(lens)]
    ref = omfa.decode_attn(bf16_np(q), k_rows, v_rows, lens, od, inp.k_scale, inp.v_scale)
    assert_close(bf16_np(out), ref, kv_dtype, "paged layer (per op)")


def test_paged_append_to_a_page_outside_the_pool_is_rejected():
    from decode_attention_10_b200 import mfa
    lens = [129, 40]
    inp = W.generate(lens, W.KV_BF16, seed=95)
    cache, k_pool, v_pool, table, need = _paged_from(inp, 128, seed=96, spare=0)
    # sequence 0 appends at row 128: its second page id now points past the pool
    bad = torch.from_numpy(table).clone()
    bad[0, 1] = k_pool.shape[0] + 7
    cache.page_table.copy_(bad.cuda())
    k_before = codes_np(k_pool).copy()
    step = GpuStep(inp)
    _, out = mfa.decode_layer(step.x, step.w_qdown, step.gamma, step.w_qup, step.w_k, step.w_v,
                              cache, step.seq_lens, ws=step.ws)
    torch.cuda.synchronize()
    assert mfa.get_error(step.ws) == 3  # MFA_ERR_CAPACITY
    kp = codes_np(k_pool)
    assert np.array_equal(kp[:, :, :][np.arange(kp.shape[0]) != table[1, 0]],
                          k_before[np.arange(kp.shape[0]) != table[1, 0]])
    assert np.isfinite(bf16_np(out)).all()  # the missing page reads as zeros


def test_cache_description_contradicting_its_table_is_reported():
    # a paged table described as contiguous (and the reverse) computes no attention, loads
    # nothing through the wrong kind of tensor map, and reports MFA_ERR_INVALID_ARG
    from decode_attention_10_b200 import mfa
    lens = [130, 7]
    inp = W.generate(lens, W.KV_BF16, seed=97)
    paged, *_ = _paged_from(inp, 128, seed=98)
    q = torch.randn(len(lens), 64, 256).to(torch.bfloat16).cuda()
    seq_lens = inp.seq_lens.cuda()
    ws = mfa.Workspace(len(lens))
    paged.desc.page_size = 0
    mfa.decode_attn(q, paged, seq_lens, ws=ws)
    assert mfa.get_error(ws) == 1
    step = GpuStep(inp)
    step.cache.desc.page_size = 128
    mfa.decode_attn(q, step.cache, seq_lens, ws=ws)
    assert mfa.get_error(ws) == 1
    step.cache.desc.page_size = 0  # described right again: the same context computes
    out = mfa.decode_attn(q, step.cache, seq_lens, ws=ws)
    assert mfa.get_error(ws) == 0
    assert np.isfinite(bf16_np(out)).all()


# ----------------------------------------------------------------------------------------
# the FP8 path: block-FP8 weights (e4m3 codes [out, in], one float32 scale per 128 x 128
# block) and FP8 activations (per row and 128 values)
# ----------------------------------------------------------------------------------------


def _q_close_fp8(q_gpu, q_ref):
    # The FP8 path decides integer codes from float inputs twice: x's codes are computed
    # identically on both sides, but c_hat comes from float32 (GPU) and float64 (oracle) sums,
    # so a one-ulp difference in a group's largest |c_hat| moves that group's scale and can
    # move every code in it by one e4m3 step (up to 2^-3 relative). Each moved code shifts q
    # by about 0.0625 |c_hat| |W_qup| (~1.4e-3); a group's 128 codes move with random signs,
    # so a few 1e-2 at most. Bound: rel-L2 1e-3, max-abs 5e-2, and at most 0.1 % of the
    # elements beyond the two-ulp bf16 bound of the bf16 path.
    ulp = np.ldexp(1.0, np.frexp(np.abs(q_ref))[1] - 8)
    off = np.abs(q_gpu - q_ref) > 2 * ulp + 1e-3
    assert off.mean() <= 1e-3, f"{off.sum()} q elements beyond two ulps"
    assert max_abs(q_gpu, q_ref) <= 5e-2
    assert rel_l2(q_gpu, q_ref) <= 1e-3


def _w8(w_bf16):
    from decode_attention_10_b200 import mfa
    codes, scales = W.quantize_w8(w_bf16)
    return mfa.BlockFP8Weight(codes.cuda(), scales.cuda()), codes.numpy(), scales.numpy()


@pytest.mark.parametrize("bsz", [1, 32, 300])
def test_query_proj_w8_matches_oracle(bsz):
    from decode_attention_10_b200 import mfa
    inp = W.generate([1] * bsz, W.KV_BF16, seed=110 + bsz)
    wq, cq, sq = _w8(inp.w_qdown)
    wu, cu, su = _w8(inp.w_qup)
    q = mfa.query_proj_w8(inp.x.cuda(), wq, inp.gamma.cuda(), wu)
    torch.cuda.synchronize()
    ow = oracle_weights(inp)
    _, q_ref = omfa.query_proj_fp8(ow["x"], cq, sq, ow["gamma"], cu, su)
    _q_close_fp8(bf16_np(q), q_ref)


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_layer_w8_matches_oracle(kv_dtype):
    from decode_attention_10_b200 import mfa
    lens = [1, 130, 300, 129, 64]
    inp = W.generate(lens, kv_dtype, seed=120)
    step = GpuStep(inp)
    k_before = [codes_np(t) for t in step.k]
    v_before = [codes_np(t) for t in step.v]
    w8s = [_w8(w) for w in (inp.w_qdown, inp.w_qup, inp.w_k, inp.w_v)]
    q = torch.empty(len(lens), 64, 256, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    run = mfa.DecodeStep(step.x, w8s[0][0], step.gamma, w8s[1][0], w8s[2][0], w8s[3][0],
                         step.cache, step.seq_lens, q, out, step.ws)
    run()
    torch.cuda.synchronize()
    assert mfa.get_error(step.ws) == 0
    od = oracle_dtype(kv_dtype)
    ow = oracle_weights(inp)
    (_, cq, sq), (_, cu, su), (_, ck, sk), (_, cv, sv) = w8s
    _, q_ref = omfa.query_proj_fp8(ow["x"], cq, sq, ow["gamma"], cu, su)
    _q_close_fp8(bf16_np(q), q_ref)
    # the appended rows: one code apart at most from the oracle's (fp32 vs float64 sums)
    k_new, v_new = omfa.fp8_project(ow["x"], ck, sk), omfa.fp8_project(ow["x"], cv, sv)
    for b, n in enumerate(lens):
        for t, want in ((step.k[b], omfa.kv_store(k_new[b], od, inp.k_scale)),
                        (step.v[b], omfa.kv_store(v_new[b], od, inp.v_scale))):
            got = codes_np(t)[n - 1].astype(np.int64)
            assert np.abs(got - want.astype(np.int64)).max() <= 1
    # end to end: the oracle's own chain (its q, its appended rows, its attention)
    k_codes = omfa.kv_store(k_new, od, inp.k_scale)
    v_codes = omfa.kv_store(v_new, od, inp.v_scale)
    k2, v2 = omfa.kv_append(k_before, v_before, [n - 1 for n in lens], k_codes, v_codes)
    ref = omfa.decode_attn(q_ref, k2, v2, lens, od, inp.k_scale, inp.v_scale)
    assert_close(bf16_np(out), ref, kv_dtype, "FP8-path layer (end to end)")
