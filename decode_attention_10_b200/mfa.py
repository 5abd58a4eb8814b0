"""Thin ctypes binding of libmfa.so (include/mfa.h): argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; this module only turns
torch tensors into pointers, picks the current CUDA stream, and raises on error statuses.
There is no fallback: if the library is missing, the first call raises.
"""

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmfa.so")

HIDDEN, Q_RANK, N_HEADS, HEAD_DIM = 7168, 2048, 64, 256
MAX_CONTEXT, MAX_BATCH = 65536, 1024
KV_BF16, KV_FP8_E4M3 = 0, 1

STATUS = {0: "MFA_OK", 1: "MFA_ERR_INVALID_ARG", 2: "MFA_ERR_UNSUPPORTED",
          3: "MFA_ERR_CAPACITY", 4: "MFA_ERR_WORKSPACE", 5: "MFA_ERR_CUDA",
          6: "MFA_ERR_EMPTY", 7: "MFA_ERR_TIMEOUT"}

class W8(ctypes.Structure):
    """mfa_w8: a block-FP8 weight (device pointers to codes and scales)."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


# name -> (restype, argtypes), mirroring include/mfa.h
_P = ctypes.c_void_p
_SIGNATURES = {
    "mfa_version": (ctypes.c_int32, []),
    "mfa_status_str": (ctypes.c_char_p, [ctypes.c_int32]),
    "mfa_kv_table_bytes": (ctypes.c_size_t, [ctypes.c_int32]),
    "mfa_kv_table_init": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int32,
                                         _P, _P, _P, _P]),
    "mfa_kv_table_init_paged": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.c_int32,
                                               ctypes.c_int32, _P, _P, ctypes.c_int32,
                                               ctypes.c_int32, _P, ctypes.c_int32, _P, _P]),
    "mfa_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32]),
    "mfa_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "mfa_get_error": (ctypes.c_int, [_P, _P]),
    "mfa_query_proj": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_float, _P, ctypes.c_int32, _P,
                                      ctypes.c_size_t, _P]),
    "mfa_kv_append": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "mfa_decode_attn": (ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, _P, ctypes.c_size_t,
                                       _P]),
    "mfa_decode_layer": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P,
                                        ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]),
    "mfa_o_proj": (ctypes.c_int, [_P, _P, _P, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "mfa_query_proj_w8": (ctypes.c_int, [_P, W8, _P, W8, ctypes.c_float, _P, ctypes.c_int32,
                                         _P, ctypes.c_size_t, _P]),
    "mfa_decode_layer_w8": (ctypes.c_int, [_P, W8, _P, W8, W8, W8, ctypes.c_float, _P, _P,
                                           ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]),
    "mfa_query_proj_noalloc": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_float, _P,
                                              ctypes.c_int32, _P]),
    "mfa_wait_selftest": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.c_uint32, _P]),
    "mfa_query_proj_noalloc_get_error": (ctypes.c_int, [_P]),
    "mfa_split_plan": (ctypes.c_int, [_P, _P, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "mfa_query_proj_noalloc_wait_selftest": (ctypes.c_int, [ctypes.c_uint32, _P]),
    "mfa_decode_layer_graph": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P,
                                              ctypes.c_float, _P, _P, _P, ctypes.c_size_t,
                                              ctypes.POINTER(ctypes.c_void_p)]),
    "mfa_decode_layer_w8_graph": (ctypes.c_int, [_P, W8, _P, W8, W8, W8, ctypes.c_float, _P,
                                                 _P, ctypes.c_float, _P, _P, _P,
                                                 ctypes.c_size_t,
                                                 ctypes.POINTER(ctypes.c_void_p)]),
    "mfa_step_graph_launch": (ctypes.c_int, [_P, _P]),
    "mfa_step_graph_destroy": (None, [_P]),
}
NOALLOC_MAX_BATCH = 32


class KvCacheDesc(ctypes.Structure):
    """mfa_kv_cache."""
    _fields_ = [("batch", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
                ("table", ctypes.c_void_p), ("page_size", ctypes.c_int32)]


class MfaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmfa.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m decode_attention_10_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise MfaError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream] = None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KV_BF16
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return KV_FP8_E4M3
    raise ValueError(f"unsupported KV dtype {t.dtype}")


class KVCache:
    """A KV cache described to the library: per-sequence K and V row buffers
    ([capacity_b, 256] CUDA tensors of bf16 or float8_e4m3fn) plus the device table.
    Keeps references to the buffers so they outlive the table."""

    def __init__(self, k: Sequence[torch.Tensor], v: Sequence[torch.Tensor],
                 k_scale: float = 1.0, v_scale: float = 1.0,
                 stream: Optional[torch.cuda.Stream] = None):
        lib = load()
        if len(k) != len(v) or not k:
            raise ValueError("need the same nonzero number of K and V buffers")
        self.k, self.v = list(k), list(v)
        self.batch = len(k)
        self.dtype = _dtype_code(k[0])
        caps = []
        for kt, vt in zip(self.k, self.v):
            if _dtype_code(kt) != self.dtype or _dtype_code(vt) != self.dtype:
                raise ValueError("mixed KV dtypes")
            if kt.dim() != 2 or kt.shape[1] != HEAD_DIM or kt.shape != vt.shape:
                raise ValueError("each K/V buffer must be [capacity, 256]")
            _ptr(kt), _ptr(vt)
            caps.append(int(kt.shape[0]))
        self.capacity = caps
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        dev = self.k[0].device
        nbytes = lib.mfa_kv_table_bytes(self.batch)
        if nbytes == 0:
            raise ValueError(f"batch {self.batch} out of range")
        self.table = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        arr = ctypes.c_void_p * self.batch
        kp = arr(*[t.data_ptr() for t in self.k])
        vp = arr(*[t.data_ptr() for t in self.v])
        cp = (ctypes.c_int32 * self.batch)(*caps)
        _check(lib.mfa_kv_table_init(self.table.data_ptr(), nbytes, self.batch, self.dtype,
                                     ctypes.cast(kp, _P), ctypes.cast(vp, _P),
                                     ctypes.cast(cp, _P), _stream(stream)),
               "mfa_kv_table_init")
        self.desc = KvCacheDesc(self.batch, self.dtype, self.k_scale, self.v_scale,
                                self.table.data_ptr(), 0)


class PagedKVCache:
    """A paged KV cache described to the library: K and V page pools ([num_pages, page_size,
    256] CUDA tensors of bf16 or float8_e4m3fn; page_size a power of two >= 64), a CUDA int32 page
    table [batch, max_pages] whose row b lists sequence b's pages in order, and the number of
    pages given to each sequence. The kernels read the page table on every call, so its
    contents may change between calls (a growing sequence's next page) without a new
    description; the pools and the table must stay in place."""

    def __init__(self, k_pool: torch.Tensor, v_pool: torch.Tensor, page_table: torch.Tensor,
                 pages_per_seq: Sequence[int], k_scale: float = 1.0, v_scale: float = 1.0,
                 stream: Optional[torch.cuda.Stream] = None):
        lib = load()
        if k_pool.dim() != 3 or k_pool.shape[2] != HEAD_DIM or k_pool.shape != v_pool.shape:
            raise ValueError("K and V pools must both be [num_pages, page_size, 256]")
        self.dtype = _dtype_code(k_pool)
        if _dtype_code(v_pool) != self.dtype:
            raise ValueError("mixed KV dtypes")
        if (page_table.dtype != torch.int32 or page_table.dim() != 2 or not page_table.is_cuda
                or not page_table.is_contiguous()):
            raise ValueError("page_table must be a contiguous CUDA int32 [batch, max_pages]")
        self.batch, max_pages = int(page_table.shape[0]), int(page_table.shape[1])
        pps = [int(n) for n in pages_per_seq]
        if len(pps) != self.batch:
            raise ValueError("one page count per sequence")
        _ptr(k_pool), _ptr(v_pool)
        self.k_pool, self.v_pool, self.page_table = k_pool, v_pool, page_table
        self.num_pages, self.page_size = int(k_pool.shape[0]), int(k_pool.shape[1])
        self.pages_per_seq = pps
        self.capacity = [n * self.page_size for n in pps]
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        nbytes = lib.mfa_kv_table_bytes(self.batch)
        if nbytes == 0:
            raise ValueError(f"batch {self.batch} out of range")
        self.table = torch.empty(nbytes, dtype=torch.uint8, device=k_pool.device)
        cp = (ctypes.c_int32 * self.batch)(*pps)
        _check(lib.mfa_kv_table_init_paged(self.table.data_ptr(), nbytes, self.batch,
                                           self.dtype, k_pool.data_ptr(), v_pool.data_ptr(),
                                           self.num_pages, self.page_size,
                                           page_table.data_ptr(), max_pages,
                                           ctypes.cast(cp, _P), _stream(stream)),
               "mfa_kv_table_init_paged")
        self.desc = KvCacheDesc(self.batch, self.dtype, self.k_scale, self.v_scale,
                                self.table.data_ptr(), self.page_size)


class BlockFP8Weight:
    """A block-FP8 projection weight for the library: e4m3 codes [out, in] (a CUDA uint8 or
    float8_e4m3fn tensor) and one float32 scale per 128 x 128 block ([out / 128, in / 128]);
    the layer multiplies with bf16(code * scale)."""

    def __init__(self, codes: torch.Tensor, scales: torch.Tensor):
        if codes.dim() != 2 or codes.element_size() != 1 or not codes.is_contiguous():
            raise ValueError("codes must be a contiguous [out, in] tensor of one-byte codes")
        out_dim, in_dim = int(codes.shape[0]), int(codes.shape[1])
        if (scales.dtype != torch.float32 or not scales.is_contiguous()
                or tuple(scales.shape) != (-(-out_dim // 128), -(-in_dim // 128))):
            raise ValueError("scales must be contiguous float32 [out / 128, in / 128]")
        _ptr(codes), _ptr(scales)
        self.codes, self.scales = codes, scales
        self.struct = W8(codes.data_ptr(), scales.data_ptr())


class Workspace:
    """Device workspace for `batch` sequences (allocated by torch, zeroed by the library)."""

    def __init__(self, batch: int, device=None, stream: Optional[torch.cuda.Stream] = None):
        lib = load()
        self.batch = int(batch)
        self.nbytes = lib.mfa_workspace_bytes(self.batch)
        if self.nbytes == 0:
            raise ValueError(f"batch {batch} out of range (or no CUDA device)")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8,
                               device=device if device is not None else "cuda")
        _check(lib.mfa_workspace_init(self.buf.data_ptr(), self.nbytes, _stream(stream)),
               "mfa_workspace_init")

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


def get_error(ws: Workspace, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronize the stream and return (and clear) the workspace's device status."""
    return load().mfa_get_error(ws.ptr, _stream(stream))


def query_proj(x, w_qdown, gamma, w_qup, eps: float = 1e-6, q_out=None, ws=None,
               stream=None) -> torch.Tensor:
    lib = load()
    bsz = int(x.shape[0])
    if q_out is None:
        q_out = torch.empty(bsz, N_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=x.device)
    ws = ws if ws is not None else Workspace(bsz, x.device)
    _check(lib.mfa_query_proj(_ptr(x), _ptr(w_qdown), _ptr(gamma), _ptr(w_qup), float(eps),
                              _ptr(q_out), bsz, ws.ptr, ws.nbytes, _stream(stream)),
           "mfa_query_proj")
    return q_out


def kv_append(x, w_k, w_v, cache: KVCache, pos: torch.Tensor, ws=None, stream=None):
    lib = load()
    ws = ws if ws is not None else Workspace(cache.batch, x.device)
    _check(lib.mfa_kv_append(_ptr(x), _ptr(w_k), _ptr(w_v), ctypes.byref(cache.desc),
                             _ptr(pos), ws.ptr, ws.nbytes, _stream(stream)),
           "mfa_kv_append")


def decode_attn(q, cache: KVCache, seq_lens: torch.Tensor, scale: float = 1.0 / 16.0,
                out=None, ws=None, stream=None) -> torch.Tensor:
    lib = load()
    if out is None:
        out = torch.empty(cache.batch, N_HEADS, HEAD_DIM, dtype=torch.bfloat16,
                          device=q.device)
    ws = ws if ws is not None else Workspace(cache.batch, q.device)
    _check(lib.mfa_decode_attn(_ptr(q), ctypes.byref(cache.desc), _ptr(seq_lens),
                               float(scale), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)),
           "mfa_decode_attn")
    return out


def decode_layer(x, w_qdown, gamma, w_qup, w_k, w_v, cache: KVCache, seq_lens,
                 eps: float = 1e-6, scale: float = 1.0 / 16.0, q_out=None, out=None,
                 ws=None, stream=None):
    """One MFA decode step; returns (q, out)."""
    lib = load()
    bsz = cache.batch
    if q_out is None:
        q_out = torch.empty(bsz, N_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=x.device)
    if out is None:
        out = torch.empty(bsz, N_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=x.device)
    ws = ws if ws is not None else Workspace(bsz, x.device)
    _check(lib.mfa_decode_layer(_ptr(x), _ptr(w_qdown), _ptr(gamma), _ptr(w_qup), _ptr(w_k),
                                _ptr(w_v), float(eps), ctypes.byref(cache.desc),
                                _ptr(seq_lens), float(scale), _ptr(q_out), _ptr(out), ws.ptr,
                                ws.nbytes, _stream(stream)),
           "mfa_decode_layer")
    return q_out, out


def o_proj(out, w_o, y=None, ws=None, stream=None) -> torch.Tensor:
    """y = bf16(out W_o): the attention output [B, 64, 256] (or [B, 16384]) projected back to
    the hidden width 7168."""
    lib = load()
    bsz = int(out.shape[0])
    if y is None:
        y = torch.empty(bsz, HIDDEN, dtype=torch.bfloat16, device=out.device)
    ws = ws if ws is not None else Workspace(bsz, out.device)
    _check(lib.mfa_o_proj(_ptr(out), _ptr(w_o), _ptr(y), bsz, ws.ptr, ws.nbytes,
                          _stream(stream)), "mfa_o_proj")
    return y


def query_proj_w8(x, w_qdown: "BlockFP8Weight", gamma, w_qup: "BlockFP8Weight",
                  eps: float = 1e-6, q_out=None, ws=None, stream=None) -> torch.Tensor:
    """mfa_query_proj with block-FP8 weights."""
    lib = load()
    bsz = int(x.shape[0])
    if q_out is None:
        q_out = torch.empty(bsz, N_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=x.device)
    ws = ws if ws is not None else Workspace(bsz, x.device)
    _check(lib.mfa_query_proj_w8(_ptr(x), w_qdown.struct, _ptr(gamma), w_qup.struct,
                                 float(eps), _ptr(q_out), bsz, ws.ptr, ws.nbytes,
                                 _stream(stream)), "mfa_query_proj_w8")
    return q_out


def query_proj_noalloc(x, w_qdown, gamma, w_qup, eps: float = 1e-6, q_out=None, stream=None):
    """mfa_query_proj without a workspace: the library's built-in scratch (batch <= 32)."""
    lib = load()
    bsz = int(x.shape[0])
    if q_out is None:
        q_out = torch.empty(bsz, N_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=x.device)
    _check(lib.mfa_query_proj_noalloc(_ptr(x), _ptr(w_qdown), _ptr(gamma), _ptr(w_qup),
                                      float(eps), _ptr(q_out), bsz, _stream(stream)),
           "mfa_query_proj_noalloc")
    return q_out


def split_plan(cache, seq_lens: torch.Tensor, grid: int, stream=None):
    """The attention's split plan as the device builds it (mfa_split_plan): returns
    (G, NT, items) with items an int tensor [n, 7] of (cta, sequence, tok0, tok1, slot,
    nsplit, split)."""
    n_max = int(grid) + cache.batch
    buf = torch.zeros(3 + 8 * n_max, dtype=torch.int32, device=seq_lens.device)
    _check(load().mfa_split_plan(ctypes.byref(cache.desc), _ptr(seq_lens), int(grid),
                                 _ptr(buf), buf.numel() * 4, _stream(stream)),
           "mfa_split_plan")
    host = buf.cpu()
    n = int(host[2])
    return int(host[0]), int(host[1]), host[3:3 + 8 * n].view(n, 8)[:, :7]


def noalloc_get_error(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status of the calls of
    query_proj_noalloc on the current device."""
    return load().mfa_query_proj_noalloc_get_error(_stream(stream))


def wait_selftest(ws: Workspace, limit_us: int = 1000, stream=None) -> None:
    """mfa_wait_selftest: enqueue a kernel whose bounded wait on a barrier that nothing
    completes gives up after limit_us; get_error(ws) then reports MFA_ERR_TIMEOUT."""
    _check(load().mfa_wait_selftest(ws.ptr, ws.nbytes, int(limit_us), _stream(stream)),
           "mfa_wait_selftest")


class DecodeStep:
    """A decode step bound to fixed buffers, for serving loops: the ctypes arguments of
    mfa_decode_layer are converted once, so each call costs one foreign call. The buffers
    (x, weights, cache, seq_lens, q_out, out, workspace) must stay alive and in place; their
    contents may change between calls (that is the point: new x, advanced seq_lens)."""

    def __init__(self, x, w_qdown, gamma, w_qup, w_k, w_v, cache: KVCache, seq_lens,
                 q_out, out, ws: Workspace, eps: float = 1e-6, scale: float = 1.0 / 16.0,
                 stream=None):
        self._lib = load()
        self._keep = (x, w_qdown, gamma, w_qup, w_k, w_v, cache, seq_lens, q_out, out, ws)
        # weights: bf16 tensors, or BlockFP8Weight (then mfa_decode_layer_w8)
        self._w8 = isinstance(w_qdown, BlockFP8Weight)
        wa = (lambda w: w.struct) if self._w8 else (lambda w: _P(_ptr(w)))
        self._fn = self._lib.mfa_decode_layer_w8 if self._w8 else self._lib.mfa_decode_layer
        self._args = (_P(_ptr(x)), wa(w_qdown), _P(_ptr(gamma)), wa(w_qup), wa(w_k), wa(w_v),
                      ctypes.c_float(eps), ctypes.byref(cache.desc), _P(_ptr(seq_lens)),
                      ctypes.c_float(scale), _P(_ptr(q_out)), _P(_ptr(out)), _P(ws.ptr),
                      ctypes.c_size_t(ws.nbytes), _P(_stream(stream)))

    def __call__(self):
        st = self._fn(*self._args)
        if st != 0:
            raise MfaError(st, "mfa_decode_layer_w8" if self._w8 else "mfa_decode_layer")


class StepGraph:
    """A decode step captured once by the library (mfa_decode_layer_graph): each call replays
    it with one graph launch (mfa_step_graph_launch) instead of the step's kernel launches,
    with results bit-identical to mfa_decode_layer's. Buffers as for DecodeStep: addresses
    fixed for the handle's life, contents free to change between calls. A replay does not
    overlap the kernel before it on the stream, so DecodeStep is the faster choice when the
    GPU, not the host, paces the loop. Captured on the current CUDA device."""

    def __init__(self, x, w_qdown, gamma, w_qup, w_k, w_v, cache: KVCache, seq_lens,
                 q_out, out, ws: Workspace, eps: float = 1e-6, scale: float = 1.0 / 16.0,
                 stream=None):
        self._lib = load()
        self._h = ctypes.c_void_p()
        self._keep = (x, w_qdown, gamma, w_qup, w_k, w_v, cache, seq_lens, q_out, out, ws)
        w8 = isinstance(w_qdown, BlockFP8Weight)
        wa = (lambda w: w.struct) if w8 else (lambda w: _P(_ptr(w)))
        fn = self._lib.mfa_decode_layer_w8_graph if w8 else self._lib.mfa_decode_layer_graph
        _check(fn(_P(_ptr(x)), wa(w_qdown), _P(_ptr(gamma)), wa(w_qup), wa(w_k), wa(w_v),
                  ctypes.c_float(eps), ctypes.byref(cache.desc), _P(_ptr(seq_lens)),
                  ctypes.c_float(scale), _P(_ptr(q_out)), _P(_ptr(out)), _P(ws.ptr),
                  ctypes.c_size_t(ws.nbytes), ctypes.byref(self._h)),
               "mfa_decode_layer_w8_graph" if w8 else "mfa_decode_layer_graph")
        self._stream = _P(_stream(stream))

    def __call__(self):
        st = self._lib.mfa_step_graph_launch(self._h, self._stream)
        if st != 0:
            raise MfaError(st, "mfa_step_graph_launch")

    def close(self):
        if self._h is not None and self._h.value is not None:
            self._lib.mfa_step_graph_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
