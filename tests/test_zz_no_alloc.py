"""mfa_query_proj_noalloc: the query projection for callers that cannot allocate device
memory (their device memory is planned up front by another component, they must not call the
allocator once running, or their plugin interface passes no workspace). It keeps its scratch
in an array inside the library instead of a caller workspace. Checked through the C ABI
against mfa_query_proj (which takes a workspace, runs the same kernels in the same order and
so must give the same bits) on calls in a row, against the float64 oracle, for every
documented rejection, and for its error read-out. This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

from decode_attention_10_b200 import workloads as W
from oracle import mfa as omfa

from mfa_util import bf16_np, oracle_weights, rel_l2

pytestmark = pytest.mark.gpu

OK, INVALID_ARG, WORKSPACE, TIMEOUT = 0, 1, 4, 7


@pytest.fixture(scope="module")
def lib():
    from decode_attention_10_b200 import build, mfa
    build.build()
    return mfa.load()


def _call_noalloc(lib, inp, q_out, stream, batch=None, eps=1e-6, x_ptr=None, q_ptr=None):
    return lib.mfa_query_proj_noalloc(
        ctypes.c_void_p(inp["x"].data_ptr() if x_ptr is None else x_ptr),
        ctypes.c_void_p(inp["w_qdown"].data_ptr()), ctypes.c_void_p(inp["gamma"].data_ptr()),
        ctypes.c_void_p(inp["w_qup"].data_ptr()), ctypes.c_float(eps),
        ctypes.c_void_p(q_out.data_ptr() if q_ptr is None else q_ptr),
        ctypes.c_int32(q_out.shape[0] if batch is None else batch), ctypes.c_void_p(stream))


def _call_with_workspace(lib, inp, q_out, stream):
    from decode_attention_10_b200 import mfa
    ws = mfa.Workspace(q_out.shape[0])
    st = lib.mfa_query_proj(
        ctypes.c_void_p(inp["x"].data_ptr()), ctypes.c_void_p(inp["w_qdown"].data_ptr()),
        ctypes.c_void_p(inp["gamma"].data_ptr()), ctypes.c_void_p(inp["w_qup"].data_ptr()),
        ctypes.c_float(1e-6), ctypes.c_void_p(q_out.data_ptr()), ctypes.c_int32(q_out.shape[0]),
        ctypes.c_void_p(ws.ptr), ctypes.c_size_t(ws.nbytes), ctypes.c_void_p(stream))
    return st, ws


def _inputs(batch, seed, x_scale=1.0):
    g = W.generate([1] * batch, W.KV_BF16, seed=seed)
    d = {k: getattr(g, k).cuda() for k in ("x", "w_qdown", "gamma", "w_qup")}
    if x_scale != 1.0:
        d["x"] = (d["x"].float() * x_scale).to(torch.bfloat16)
    d["host"] = g
    return d


def _q_close_to_oracle(q_gpu, inp):
    # the oracle's query path on the same bytes (c_hat and q rounded to bf16 as stored); q is
    # held to two bf16 ulps of the reference plus 1e-3 per element and rel-L2 1e-3
    w = oracle_weights(inp["host"])
    x = bf16_np(inp["x"])
    _, ref = omfa.query_proj(x, w["w_qdown"], w["gamma"], w["w_qup"])
    q = bf16_np(q_gpu)
    ulp = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 8)
    assert (np.abs(q - ref) <= 2 * ulp + 1e-3).all()
    assert rel_l2(q, ref) <= 1e-3


def test_noalloc_matches_workspace_call_twice_in_a_row(lib):
    from decode_attention_10_b200 import mfa
    stream = torch.cuda.current_stream().cuda_stream
    assert mfa.noalloc_get_error() == OK
    # calls in a row on the shared scratch: a full batch with inputs 100 times larger, then
    # a small batch, then the full batch again. Partials or c_hat rows the first call left
    # behind would change the later results visibly; every result must equal, bit for bit,
    # the workspace call on the same inputs (same kernels, same order), and the oracle.
    for batch, seed, scale in ((32, 41, 100.0), (5, 42, 1.0), (32, 43, 1.0)):
        inp = _inputs(batch, seed, scale)
        q_na = torch.empty(batch, 64, 256, dtype=torch.bfloat16, device="cuda")
        q_ws = torch.empty_like(q_na)
        assert _call_noalloc(lib, inp, q_na, stream) == OK
        st, ws = _call_with_workspace(lib, inp, q_ws, stream)
        assert st == OK
        torch.cuda.synchronize()
        assert torch.equal(q_na, q_ws), f"batch {batch}: differs from the workspace call"
        assert torch.isfinite(q_na.float()).all()
        _q_close_to_oracle(q_na, inp)
    assert mfa.noalloc_get_error() == OK


@pytest.mark.parametrize("case", ["batch_over_limit", "batch_zero", "eps_zero", "null_q_out",
                                  "misaligned_x"])
def test_noalloc_rejects_bad_arguments_and_enqueues_nothing(lib, case):
    stream = torch.cuda.current_stream().cuda_stream
    batch = 33 if case == "batch_over_limit" else 4
    inp = _inputs(batch, 44)
    q = torch.zeros(batch, 64, 256, dtype=torch.bfloat16, device="cuda")
    kw, want = {}, INVALID_ARG
    if case == "batch_over_limit":
        want = WORKSPACE  # the built-in scratch holds at most 32 rows
    elif case == "batch_zero":
        kw["batch"] = 0
    elif case == "eps_zero":
        kw["eps"] = 0.0
    elif case == "null_q_out":
        kw["q_ptr"] = 0
    elif case == "misaligned_x":
        kw["x_ptr"] = inp["x"].data_ptr() + 2
    assert _call_noalloc(lib, inp, q, stream, **kw) == want
    torch.cuda.synchronize()
    assert (q.float() == 0).all()  # nothing was enqueued


def test_noalloc_error_word_is_reported_once_and_cleared(lib):
    from decode_attention_10_b200 import mfa
    stream = torch.cuda.current_stream().cuda_stream
    assert mfa.noalloc_get_error() == OK
    # a bounded wait that expires on the built-in scratch's error word, as one inside the
    # projection kernels would
    assert lib.mfa_query_proj_noalloc_wait_selftest(ctypes.c_uint32(2000),
                                                    ctypes.c_void_p(stream)) == OK
    assert lib.mfa_query_proj_noalloc_wait_selftest(ctypes.c_uint32(0),
                                                    ctypes.c_void_p(stream)) == INVALID_ARG
    assert mfa.noalloc_get_error() == TIMEOUT
    assert mfa.noalloc_get_error() == OK  # read once, then cleared
    # the entry point still computes the same bits as the workspace call afterwards
    inp = _inputs(8, 45)
    q_na = torch.empty(8, 64, 256, dtype=torch.bfloat16, device="cuda")
    q_ws = torch.empty_like(q_na)
    assert _call_noalloc(lib, inp, q_na, stream) == OK
    assert _call_with_workspace(lib, inp, q_ws, stream)[0] == OK
    torch.cuda.synchronize()
    assert torch.equal(q_na, q_ws)
    assert mfa.noalloc_get_error() == OK
