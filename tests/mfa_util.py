"""Shared helpers of the tests: moving seeded inputs to the GPU, feeding the oracle the same
bytes, and the tolerance checks."""

import numpy as np
import torch

from decode_attention_10_b200 import workloads as W
from oracle import codecs
from oracle import mfa as omfa

# Tolerances for bf16 outputs: relative L2 error and max abs error (bf16 KV), max abs error
# for FP8 KV (against an oracle that reads the same stored codes).
REL_L2 = 5e-3
MAX_ABS_BF16 = 2e-2
MAX_ABS_FP8 = 3e-2


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> float64 values, decoded by the oracle's own codec."""
    bits = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return codecs.bf16_decode(bits)


def codes_np(t: torch.Tensor) -> np.ndarray:
    """Cache tensor -> its raw codes (uint16 bf16 bits or uint8 e4m3 codes)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.uint8).numpy()


def oracle_dtype(kv_dtype: str) -> str:
    return omfa.KV_BF16 if kv_dtype == W.KV_BF16 else omfa.KV_FP8


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def assert_close(gpu, ref, kv_dtype=W.KV_BF16, what=""):
    r, m = rel_l2(gpu, ref), max_abs(gpu, ref)
    lim = MAX_ABS_FP8 if kv_dtype == W.KV_FP8 else MAX_ABS_BF16
    assert r <= REL_L2 and m <= lim, f"{what}: rel_l2={r:.3e} max_abs={m:.3e}"
    return r, m


class GpuStep:
    """The inputs of one decode step on the GPU, with the library's KV table/workspace."""

    def __init__(self, inp: W.Inputs, device="cuda"):
        from decode_attention_10_b200 import mfa
        self.inp = inp
        dev = torch.device(device)
        self.x = inp.x.to(dev)
        self.w_qdown = inp.w_qdown.to(dev)
        self.gamma = inp.gamma.to(dev)
        self.w_qup = inp.w_qup.to(dev)
        self.w_k = inp.w_k.to(dev)
        self.w_v = inp.w_v.to(dev)
        if inp.k_buffer is not None:
            self.k_buffer = inp.k_buffer.to(dev)
            self.v_buffer = inp.v_buffer.to(dev)
            self.k = [self.k_buffer[b] for b in range(inp.batch)]
            self.v = [self.v_buffer[b] for b in range(inp.batch)]
        else:
            self.k_buffer = self.v_buffer = None
            self.k = [t.to(dev) for t in inp.k_cache]
            self.v = [t.to(dev) for t in inp.v_cache]
        self.seq_lens = inp.seq_lens.to(dev)
        self.cache = mfa.KVCache(self.k, self.v, inp.k_scale, inp.v_scale)
        self.ws = mfa.Workspace(inp.batch, dev)

    def layer(self, eps=1e-6, scale=1.0 / 16.0):
        from decode_attention_10_b200 import mfa
        return mfa.decode_layer(self.x, self.w_qdown, self.gamma, self.w_qup, self.w_k,
                                self.w_v, self.cache, self.seq_lens, eps=eps, scale=scale,
                                ws=self.ws)


def oracle_weights(inp: W.Inputs):
    return dict(x=bf16_np(inp.x), w_qdown=bf16_np(inp.w_qdown), gamma=bf16_np(inp.gamma),
                w_qup=bf16_np(inp.w_qup), w_k=bf16_np(inp.w_k), w_v=bf16_np(inp.w_v))
