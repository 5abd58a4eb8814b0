"""The analytic step cost (max(attention compute, KV access) + linear projections, the Step-3
pages' cost framing): its counts against closed forms and against bench.py's own byte
counts, and its roofline arithmetic."""

import os
import sys

import pytest

from decode_attention_10_b200 import cost_model as cm
from decode_attention_10_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_weight_bytes_match_the_layer_shapes():
    # W_qdown [7168, 2048], W_qup [2048, 16384], W_k and W_v [7168, 256], bf16
    assert cm.WEIGHT_BYTES == 103_809_024
    assert cm.ATTN_FLOPS_PER_POSITION == 65_536  # 2 (q.k) + 2 (p.v) flops x 64 heads x 256


def test_counts_closed_form():
    c = cm.step_counts([4096] * 32, "bf16")
    assert c.positions == 32 * 4096
    assert c.attn_bytes == 2 * 512 * 32 * 4096 + 2 * 32 * 16384 * 2  # K+V rows, q in, out
    assert c.attn_flops == 65_536 * 32 * 4096
    assert c.linear_flops == 2 * 32 * (7168 * 2048 + 2048 * 16384 + 2 * 7168 * 256)
    f = cm.step_counts([4096] * 32, "fp8_e4m3")
    assert f.attn_bytes - 2 * 32 * 16384 * 2 == (c.attn_bytes - 2 * 32 * 16384 * 2) // 2


def test_attention_bytes_agree_with_bench():
    sys.path.insert(0, ROOT)
    import bench
    for lens, dt in (([1, 130, 300], W.KV_BF16), ([7, 2000], W.KV_FP8)):
        inp = W.generate(lens, dt, seed=3)
        assert cm.step_counts(lens, dt).attn_bytes == bench.attention_bytes(inp)
    assert cm.WEIGHT_BYTES == bench.WEIGHT_BYTES


def test_roofline_bound_and_times():
    c = cm.step_counts([4096] * 32, "bf16")
    t = cm.step_times(c, hbm_gbs=1000.0, tensor_tflops=1000.0)
    assert t.attn_bound == "hbm" and t.linear_bound == "hbm"
    assert t.attn_s == pytest.approx(c.attn_bytes / 1e12)
    assert t.step_s == pytest.approx(t.attn_s + t.linear_s)
    assert t.per_token_s == pytest.approx(t.step_s / 32)
    # a slow tensor core makes the attention compute-bound
    slow = cm.step_times(c, hbm_gbs=1000.0, tensor_tflops=1.0)
    assert slow.attn_bound == "tensor" and slow.attn_s == pytest.approx(c.attn_flops / 1e12)
    r = cm.layer_roofline(c, 2 * t.step_s, 1000.0, 1000.0)
    assert r["frac"] == pytest.approx(0.5)


def test_workload_lens_match_the_generator():
    w = W.workload(4)
    assert cm.step_counts(W.workload_lens(w), w.kv_dtype).batch == 16
    assert W.workload_lens(w) == W.ragged_lengths(16, 1004)
    assert W.workload_lens(W.workload(1)) == [4096] * 32


def test_o_proj_counts_and_stack_model():
    base = cm.step_counts([4096] * 32, "bf16")
    full = cm.step_counts([4096] * 32, "bf16", o_proj=True)
    assert cm.O_PROJ_ELEMS == 16384 * 7168
    assert full.linear_flops - base.linear_flops == 2 * 32 * 16384 * 7168
    # W_o once (234,881,024 B) + out read + y written
    assert full.linear_bytes - base.linear_bytes == 234_881_024 + 32 * 16384 * 2 + 32 * 7168 * 2
    assert full.attn_bytes == base.attn_bytes
    t = cm.step_times(full, 1000.0, 1000.0)
    r = cm.stack_roofline(full, 61, 61 * 2 * t.step_s, 1000.0, 1000.0)
    assert r["frac"] == pytest.approx(0.5)
    assert r["model_us_per_layer"] == pytest.approx(t.step_s * 1e6)
    assert r["measured_us_per_layer"] == pytest.approx(2 * t.step_s * 1e6)
