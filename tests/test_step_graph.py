"""The captured decode step (mfa_decode_layer_graph / mfa_step_graph_launch, include/mfa.h):
a replay must give exactly what the direct call gives on the same buffers (the same kernels
with the same arguments), read the buffers' contents at replay time (a new x and new
lengths in the same buffers), and stay within the oracle's tolerances."""

import numpy as np
import pytest
import torch

from decode_attention_10_b200 import workloads as W
from oracle import mfa as omfa

from mfa_util import GpuStep, assert_close, bf16_np, codes_np, oracle_dtype, oracle_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from decode_attention_10_b200 import build, mfa
    build.build()
    mfa.load()


def _weights(step, w8):
    from decode_attention_10_b200 import mfa
    if not w8:
        return step.w_qdown, step.gamma, step.w_qup, step.w_k, step.w_v
    out = []
    for w in (step.w_qdown, step.w_qup, step.w_k, step.w_v):
        codes, scales = W.quantize_w8(w.cpu())
        out.append(mfa.BlockFP8Weight(codes.cuda(), scales.cuda()))
    return out[0], step.gamma, out[1], out[2], out[3]


def _state(step, q, out):
    torch.cuda.synchronize()
    return (q.clone(), out.clone(), [t.clone() for t in step.k], [t.clone() for t in step.v])


def _restore(step, k0, v0):
    for t, s in zip(step.k + step.v, k0 + v0):
        t.copy_(s)
    torch.cuda.synchronize()


def _same(a, b):
    qa, oa, ka, va = a
    qb, ob, kb, vb = b
    assert torch.equal(qa, qb), "q differs from the direct call"
    assert torch.equal(oa, ob), "attention output differs from the direct call"
    for x, y in zip(ka + va, kb + vb):
        assert torch.equal(x, y), "cache differs from the direct call"


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
@pytest.mark.parametrize("w8", [False, True], ids=["bf16_weights", "fp8_weights"])
def test_replay_bit_identical_to_direct_call(kv_dtype, w8):
    from decode_attention_10_b200 import mfa
    lens = [1, 130, 300, 129, 64]
    inp = W.generate(lens, kv_dtype, seed=140, capacity=[n + 3 for n in lens])
    step = GpuStep(inp)
    wts = _weights(step, w8)
    q = torch.empty(len(lens), 64, 256, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    args = (step.x, *wts, step.cache, step.seq_lens, q, out, step.ws)
    direct = mfa.DecodeStep(*args)
    graph = mfa.StepGraph(*args)
    k0, v0 = [t.clone() for t in step.k], [t.clone() for t in step.v]

    # the inputs of the capture
    direct()
    want = _state(step, q, out)
    _restore(step, k0, v0)
    graph()
    _same(_state(step, q, out), want)
    assert mfa.get_error(step.ws) == 0

    # new contents in the same buffers: another x, every sequence two positions longer (its
    # new rows appended at the new last position), so the plan changes too
    x2 = W.generate(lens, kv_dtype, seed=141).x
    lens2 = [n + 2 for n in lens]
    step.x.copy_(x2.cuda())
    step.seq_lens.copy_(torch.tensor(lens2, dtype=torch.int32))
    _restore(step, k0, v0)
    direct()
    want2 = _state(step, q, out)
    _restore(step, k0, v0)
    graph()
    got2 = _state(step, q, out)
    _same(got2, want2)
    assert not torch.equal(want2[1], want[1])
    assert mfa.get_error(step.ws) == 0

    if not w8:
        # and the replay against the oracle: q from the new x, attention over the cache the
        # replay left (its appended rows included) at the new lengths
        ow = oracle_weights(inp)
        _, q_ref = omfa.query_proj(bf16_np(x2), ow["w_qdown"], ow["gamma"], ow["w_qup"])
        q_np = bf16_np(got2[0])
        assert np.abs(q_np - q_ref).max() <= 5e-2
        od = oracle_dtype(kv_dtype)
        ref = omfa.decode_attn(q_np, [codes_np(t) for t in got2[2]],
                               [codes_np(t) for t in got2[3]], lens2, od, inp.k_scale,
                               inp.v_scale)
        assert_close(bf16_np(got2[1]), ref, kv_dtype, "replayed step (per op)")
    graph.close()


def test_capture_rejects_bad_arguments_and_leaves_no_handle():
    import ctypes

    from decode_attention_10_b200 import mfa
    lib = mfa.load()
    inp = W.generate([5, 9], W.KV_BF16, seed=142)
    step = GpuStep(inp)
    q = torch.empty(2, 64, 256, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    P = ctypes.c_void_p
    h = ctypes.c_void_p(1234)
    base = [P(step.x.data_ptr()), P(step.w_qdown.data_ptr()), P(step.gamma.data_ptr()),
            P(step.w_qup.data_ptr()), P(step.w_k.data_ptr()), P(step.w_v.data_ptr()),
            ctypes.c_float(1e-6), ctypes.byref(step.cache.desc), P(step.seq_lens.data_ptr()),
            ctypes.c_float(1 / 16), P(q.data_ptr()), P(out.data_ptr()), P(step.ws.ptr),
            ctypes.c_size_t(step.ws.nbytes)]
    for i, bad in ((6, ctypes.c_float(0.0)), (0, P(step.x.data_ptr() + 2)),
                   (13, ctypes.c_size_t(64))):
        a = list(base)
        a[i] = bad
        st = lib.mfa_decode_layer_graph(*a, ctypes.byref(h))
        assert st in (1, 4), mfa.STATUS.get(st, st)
        assert h.value is None, "a rejected capture must leave no handle"
        h = ctypes.c_void_p(1234)
    # a good capture, replayed twice back to back
    assert lib.mfa_decode_layer_graph(*base, ctypes.byref(h)) == 0
    assert h.value is not None
    s = torch.cuda.current_stream().cuda_stream
    assert lib.mfa_step_graph_launch(h, P(s)) == 0
    assert lib.mfa_step_graph_launch(h, P(s)) == 0
    torch.cuda.synchronize()
    assert mfa.get_error(step.ws) == 0
    lib.mfa_step_graph_destroy(h)


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_FP8])
def test_chained_steps_on_one_workspace_match_isolated_steps(kv_dtype):
    # Consecutive steps on a stream overlap through programmatic dependent launch (each
    # step's first kernel streams weights while the previous step's combine runs) and share
    # the workspace. Two input sets with different x and lengths (so different split plans),
    # run A, B, A, B back to back -- direct calls and one CUDA graph of the four calls --
    # must leave exactly the outputs of isolated calls.
    from decode_attention_10_b200 import mfa
    sets = []
    ws = None
    for lens, seed in (([1, 130, 300, 129], 150), ([257, 64, 1000, 5], 151)):
        inp = W.generate(lens, kv_dtype, seed=seed)
        st = GpuStep(inp)
        if ws is None:
            ws = st.ws
        q = torch.empty(len(lens), 64, 256, dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(q)
        st.call = mfa.DecodeStep(st.x, st.w_qdown, st.gamma, st.w_qup, st.w_k, st.w_v,
                                 st.cache, st.seq_lens, q, out, ws)
        st.q_buf, st.out_buf = q, out
        sets.append(st)
    ref = []
    for st in sets:  # isolated: each call alone on an idle stream (the append is idempotent)
        torch.cuda.synchronize()
        st.call()
        torch.cuda.synchronize()
        ref.append((st.q_buf.clone(), st.out_buf.clone()))
    assert mfa.get_error(ws) == 0

    def check(where):
        torch.cuda.synchronize()
        for st, (q0, o0) in zip(sets, ref):
            assert torch.equal(st.q_buf, q0), f"{where}: q differs from the isolated call"
            assert torch.equal(st.out_buf, o0), f"{where}: output differs from the isolated call"
        assert mfa.get_error(ws) == 0

    for st in sets:
        st.q_buf.zero_()
        st.out_buf.zero_()
    for st in sets + sets:  # direct calls, back to back
        st.call()
    check("direct chain")

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        for st in sets:
            st.gcall = mfa.DecodeStep(st.x, st.w_qdown, st.gamma, st.w_qup, st.w_k, st.w_v,
                                      st.cache, st.seq_lens, st.q_buf, st.out_buf, ws,
                                      stream=side)
        with torch.cuda.graph(g, stream=side):
            for st in sets + sets:
                st.gcall()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for st in sets:
        st.q_buf.zero_()
        st.out_buf.zero_()
    g.replay()
    check("graph of four chained steps")
    del g
