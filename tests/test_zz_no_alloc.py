"""mfa_query_proj_noalloc: the query projection for callers that cannot allocate device
memory, using the library's built-in scratch array instead of a caller workspace. Checked
through the C ABI against mfa_query_proj (which takes a workspace) on two calls in a row,
and for its batch limit. This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

from decode_attention_10_b200 import workloads as W

from mfa_util import MAX_ABS_BF16, REL_L2, bf16_np, max_abs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from decode_attention_10_b200 import build, mfa
    build.build()
    return mfa.load()


def _call_noalloc(lib, inp, q_out, stream):
    return lib.mfa_query_proj_noalloc(
        ctypes.c_void_p(inp["x"].data_ptr()), ctypes.c_void_p(inp["w_qdown"].data_ptr()),
        ctypes.c_void_p(inp["gamma"].data_ptr()), ctypes.c_void_p(inp["w_qup"].data_ptr()),
        ctypes.c_float(1e-6), ctypes.c_void_p(q_out.data_ptr()), ctypes.c_int32(q_out.shape[0]),
        ctypes.c_void_p(stream))


def _call_with_workspace(lib, inp, q_out, stream):
    from decode_attention_10_b200 import mfa
    ws = mfa.Workspace(q_out.shape[0])
    st = lib.mfa_query_proj(
        ctypes.c_void_p(inp["x"].data_ptr()), ctypes.c_void_p(inp["w_qdown"].data_ptr()),
        ctypes.c_void_p(inp["gamma"].data_ptr()), ctypes.c_void_p(inp["w_qup"].data_ptr()),
        ctypes.c_float(1e-6), ctypes.c_void_p(q_out.data_ptr()), ctypes.c_int32(q_out.shape[0]),
        ctypes.c_void_p(ws.ptr), ctypes.c_size_t(ws.nbytes), ctypes.c_void_p(stream))
    return st, ws


def _inputs(batch, seed):
    g = W.generate([1] * batch, W.KV_BF16, seed=seed)
    return {k: getattr(g, k).cuda() for k in ("x", "w_qdown", "gamma", "w_qup")}


def test_noalloc_matches_workspace_call_twice_in_a_row(lib):
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row with different inputs and batch sizes: the second call must not
    # see anything the first one left in the shared scratch
    for batch, seed in ((32, 41), (5, 42)):
        inp = _inputs(batch, seed)
        q_na = torch.empty(batch, 64, 256, dtype=torch.bfloat16, device="cuda")
        q_ws = torch.empty_like(q_na)
        assert _call_noalloc(lib, inp, q_na, stream) == 0
        st, ws = _call_with_workspace(lib, inp, q_ws, stream)
        assert st == 0
        torch.cuda.synchronize()
        a, b = bf16_np(q_na), bf16_np(q_ws)
        assert rel_l2(a, b) <= REL_L2 and max_abs(a, b) <= MAX_ABS_BF16
        assert np.isfinite(a).all()


def test_noalloc_rejects_batch_above_its_limit(lib):
    stream = torch.cuda.current_stream().cuda_stream
    inp = _inputs(33, 43)
    q = torch.zeros(33, 64, 256, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, inp, q, stream) == 4  # MFA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (q.float() == 0).all()  # nothing was enqueued
