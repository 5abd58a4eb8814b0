"""The C-ABI library without a GPU: it loads, exports every symbol include/mfa.h declares,
and rejects bad arguments with the documented status before touching the device."""

import ctypes
import os
import re

import pytest

from decode_attention_10_b200 import mfa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mfa.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MFA_API\s+[\w\s\*]+?\b(mfa_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from decode_attention_10_b200 import build
    build.build()
    return mfa.load()


def test_header_declares_the_four_layer_calls():
    names = declared_functions()
    for n in ("mfa_query_proj", "mfa_kv_append", "mfa_decode_attn", "mfa_decode_layer"):
        assert n in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in mfa._SIGNATURES, f"binding lacks {name}"


def test_header_constants_match_binding_and_pages():
    import json
    text = open(HEADER).read()
    consts = dict(re.findall(r"#define (MFA_\w+) (\d+)", text))
    with open(os.path.join(ROOT, "tests", "golden", "page_dims.json")) as f:
        dims = json.load(f)
    assert int(consts["MFA_HIDDEN"]) == dims["hidden"] == mfa.HIDDEN
    assert int(consts["MFA_Q_RANK"]) == dims["q_rank"] == mfa.Q_RANK
    assert int(consts["MFA_N_HEADS"]) == dims["n_heads"] == mfa.N_HEADS
    assert int(consts["MFA_HEAD_DIM"]) == dims["head_dim"] == mfa.HEAD_DIM
    assert int(consts["MFA_MAX_CONTEXT"]) == dims["max_context"] == mfa.MAX_CONTEXT
    assert int(consts["MFA_MAX_BATCH"]) == mfa.MAX_BATCH


def test_version_and_status_strings(lib):
    assert lib.mfa_version() >= 100
    for code, name in mfa.STATUS.items():
        assert lib.mfa_status_str(code).decode() == name
    assert lib.mfa_status_str(99).decode() == "MFA_ERR_UNKNOWN"


def test_table_bytes_range(lib):
    assert lib.mfa_kv_table_bytes(0) == 0
    assert lib.mfa_kv_table_bytes(mfa.MAX_BATCH + 1) == 0
    assert lib.mfa_kv_table_bytes(1) == 384
    assert lib.mfa_kv_table_bytes(16) == 16 * 384


def test_invalid_arguments_are_rejected_before_any_device_work(lib):
    P = ctypes.c_void_p
    fake = P(4096)  # never dereferenced: every call below fails its host-side checks
    # batch out of range
    assert lib.mfa_query_proj(fake, fake, fake, fake, 1e-6, fake, 0, fake, 1 << 30, None) == 1
    assert lib.mfa_query_proj(fake, fake, fake, fake, 1e-6, fake, 1025, fake, 1 << 30,
                              None) == 1
    # eps must be > 0
    assert lib.mfa_query_proj(fake, fake, fake, fake, 0.0, fake, 4, fake, 1 << 30, None) == 1
    # null / misaligned pointers
    assert lib.mfa_query_proj(None, fake, fake, fake, 1e-6, fake, 4, fake, 1 << 30, None) == 1
    assert lib.mfa_query_proj(P(4097), fake, fake, fake, 1e-6, fake, 4, fake, 1 << 30,
                              None) == 1
    # KV cache description checks
    kv = mfa.KvCacheDesc(0, 0, 1.0, 1.0, 4096)
    assert lib.mfa_decode_attn(fake, ctypes.byref(kv), fake, 0.0625, fake, fake, 1 << 30,
                               None) == 1
    kv = mfa.KvCacheDesc(4, 7, 1.0, 1.0, 4096)
    assert lib.mfa_decode_attn(fake, ctypes.byref(kv), fake, 0.0625, fake, fake, 1 << 30,
                               None) == 2
    kv = mfa.KvCacheDesc(4, 1, 0.0, 1.0, 4096)  # FP8 needs positive scales
    assert lib.mfa_decode_attn(fake, ctypes.byref(kv), fake, 0.0625, fake, fake, 1 << 30,
                               None) == 1
    for ps in (32, 100, 192):  # a stated page size must be 0 or a power of two >= 64
        kv = mfa.KvCacheDesc(4, 0, 1.0, 1.0, 4096, ps)
        assert lib.mfa_decode_attn(fake, ctypes.byref(kv), fake, 0.0625, fake, fake, 1 << 30,
                                   None) == 1
    kv = mfa.KvCacheDesc(4, 0, 1.0, 1.0, 4096 + 64)  # table must be 128-byte aligned
    assert lib.mfa_kv_append(fake, fake, fake, ctypes.byref(kv), fake, fake, 1 << 30,
                             None) == 1
    assert lib.mfa_decode_attn(fake, None, fake, 0.0625, fake, fake, 1 << 30, None) == 1
    kv = mfa.KvCacheDesc(4, 0, 1.0, 1.0, 4096)
    assert lib.mfa_decode_layer(fake, fake, fake, fake, fake, fake, 1e-6, ctypes.byref(kv),
                                fake, -1.0, fake, fake, fake, 1 << 30, None) == 1
    # output projection: batch range, null / misaligned pointers
    assert lib.mfa_o_proj(fake, fake, fake, 0, fake, 1 << 30, None) == 1
    assert lib.mfa_o_proj(fake, fake, fake, 1025, fake, 1 << 30, None) == 1
    assert lib.mfa_o_proj(None, fake, fake, 4, fake, 1 << 30, None) == 1
    assert lib.mfa_o_proj(fake, fake, P(4104), 4, fake, 1 << 30, None) == 1
    # paged table init: page sizes that are not a power of two >= 64, bad page counts
    pages = (ctypes.c_int32 * 2)(1, 1)
    for ps in (0, 32, 96, 192):
        assert lib.mfa_kv_table_init_paged(P(4096), 1 << 20, 2, 0, fake, fake, 8, ps, fake, 4,
                                           pages, None) == 2
    bad_pages = (ctypes.c_int32 * 2)(1, 5)  # more than max_pages
    assert lib.mfa_kv_table_init_paged(P(4096), 1 << 20, 2, 0, fake, fake, 8, 128, fake, 4,
                                       bad_pages, None) == 1
    assert lib.mfa_kv_table_init_paged(P(4096), 1 << 20, 2, 0, None, fake, 8, 128, fake, 4,
                                       pages, None) == 1
    # table init: bad batch, null arrays, unknown dtype, table too small, capacity range
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    caps = (ctypes.c_int32 * 2)(16, 16)
    cap_bad = (ctypes.c_int32 * 2)(16, 65537)
    t = P(4096)
    assert lib.mfa_kv_table_init(t, 1 << 20, 0, 0, arr, arr, caps, None) == 1
    assert lib.mfa_kv_table_init(t, 1 << 20, 2, 0, None, arr, caps, None) == 1
    assert lib.mfa_kv_table_init(t, 1 << 20, 2, 5, arr, arr, caps, None) == 2
    assert lib.mfa_kv_table_init(t, 100, 2, 0, arr, arr, caps, None) == 4
    assert lib.mfa_kv_table_init(t, 1 << 20, 2, 0, arr, arr, cap_bad, None) == 1
    mis = (ctypes.c_void_p * 2)(4096, 8200)
    assert lib.mfa_kv_table_init(t, 1 << 20, 2, 0, mis, arr, caps, None) == 1
    assert lib.mfa_workspace_init(P(4100), 1024, None) == 1
    assert lib.mfa_get_error(None, None) == 1


def test_captured_step_arguments_are_rejected_before_any_device_work(lib):
    P = ctypes.c_void_p
    fake = P(4096)
    kv = mfa.KvCacheDesc(4, 0, 1.0, 1.0, 4096)
    h = ctypes.c_void_p(1234)
    # no place for the handle
    assert lib.mfa_decode_layer_graph(fake, fake, fake, fake, fake, fake, 1e-6,
                                      ctypes.byref(kv), fake, 0.0625, fake, fake, fake,
                                      1 << 30, None) == 1
    # a rejected argument leaves a NULL handle (scale, a misaligned x, a bad cache)
    for scale, x, desc in ((-1.0, fake, kv), (0.0625, P(4098), kv),
                           (0.0625, fake, mfa.KvCacheDesc(0, 0, 1.0, 1.0, 4096))):
        assert lib.mfa_decode_layer_graph(x, fake, fake, fake, fake, fake, 1e-6,
                                          ctypes.byref(desc), fake, scale, fake, fake, fake,
                                          1 << 30, ctypes.byref(h)) == 1
        assert h.value is None
        h = ctypes.c_void_p(1234)
    w = mfa.W8(4096, 4096)
    bad_w = mfa.W8(4096, None)  # FP8 weights need their scales
    assert lib.mfa_decode_layer_w8_graph(fake, w, fake, w, bad_w, w, 1e-6, ctypes.byref(kv),
                                         fake, 0.0625, fake, fake, fake, 1 << 30,
                                         ctypes.byref(h)) == 1
    assert h.value is None
    assert lib.mfa_step_graph_launch(None, None) == 1
    lib.mfa_step_graph_destroy(None)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(mfa, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mfa.load(str(tmp_path / "nope.so"))


def test_header_compiles_as_c99_and_the_library_links_from_c(lib, tmp_path):
    # the boundary needs no Python and no torch: a C99 program includes the header, links
    # libmfa.so and gets the documented statuses for calls rejected before any device work
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi_check.c"
    src.write_text(r"""
#include <stdio.h>
#include "mfa.h"
int main(void) {
  void* fake = (void*)4096;
  mfa_kv_cache kv = {4, MFA_KV_BF16, 1.0f, 1.0f, fake, 0};
  mfa_step_graph* g = (mfa_step_graph*)fake;
  int bad = 0;
  bad |= mfa_version() < 100;
  bad |= mfa_query_proj(fake, fake, fake, fake, 0.0f, fake, 4, fake, 1u << 30, 0) !=
         MFA_ERR_INVALID_ARG;
  bad |= mfa_decode_attn(fake, 0, fake, 0.0625f, fake, fake, 1u << 30, 0) !=
         MFA_ERR_INVALID_ARG;
  bad |= mfa_decode_layer_graph(fake, fake, fake, fake, fake, fake, 1e-6f, &kv, fake, -1.0f,
                                fake, fake, fake, 1u << 30, &g) != MFA_ERR_INVALID_ARG;
  bad |= g != 0;
  bad |= mfa_step_graph_launch(0, 0) != MFA_ERR_INVALID_ARG;
  mfa_step_graph_destroy(0);
  printf("%s %s\n", bad ? "FAIL" : "OK", mfa_status_str(MFA_ERR_WORKSPACE));
  return bad;
}
""")
    libdir = os.path.join(ROOT, "decode_attention_10_b200")
    exe = tmp_path / "abi_check"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmfa",
                    "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.split() == ["OK", "MFA_ERR_WORKSPACE"]
