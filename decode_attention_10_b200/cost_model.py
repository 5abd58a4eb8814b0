"""Analytic cost of one MFA decode step on a GPU, in the Step-3 pages' framing.

The pages (bud-325 summary, "Method": the cost analysis of their section 4) factor the
per-token decoding cost of a layer into max(attention compute, KV memory access) + the linear
projections (+ the FFN, which is not part of this step), each part taken at the roofline of the
hardware that runs it. For one step of the MFA attention layer over a batch:

  attention:  flops = 4 * heads * head_dim flops per (sequence, attended position)
                      (q.k and p.v, 2 flops each, for the 64 heads of dimension 256)
              bytes = every attended K and V row once + q read + out written
              time  = max(flops / tensor peak, bytes / HBM peak)
  linear:     flops = 2 * batch * (7168 * 2048 + 2048 * 16384 + 2 * 7168 * 256)
              bytes = the bf16 weights once (103,809,024 B) + x read + q written + the appended
                      K/V rows
              time  = max(flops / tensor peak, bytes / HBM peak)
  step        = attention + linear   (the two do not overlap in the model: the attention needs q)

`layer_roofline` divides the modelled step time by a measured one: the fraction of the
hardware's roofline the implementation reaches for the whole step. The pages price the parts in
dollars per million tokens on named GPUs; with no B200 price on the pages, `gpu_seconds_per_m`
reports the GPU time per million tokens instead.
"""

from dataclasses import dataclass
from typing import Iterable, Optional

HIDDEN, Q_RANK, HEADS, HEAD_DIM = 7168, 2048, 64, 256
Q_WIDTH = HEADS * HEAD_DIM
WEIGHT_ELEMS = HIDDEN * Q_RANK + Q_RANK * Q_WIDTH + 2 * HIDDEN * HEAD_DIM
WEIGHT_BYTES = 2 * WEIGHT_ELEMS  # bf16
ATTN_FLOPS_PER_POSITION = 4 * HEADS * HEAD_DIM  # 65,536
O_PROJ_ELEMS = Q_WIDTH * HIDDEN  # the output projection W_o [16384, 7168]


@dataclass
class StepCounts:
    batch: int
    positions: int          # sum over sequences of attended positions
    attn_flops: float
    attn_bytes: float
    linear_flops: float
    linear_bytes: float


@dataclass
class StepTimes:
    attn_s: float
    linear_s: float
    step_s: float
    attn_bound: str         # "hbm" or "tensor"
    linear_bound: str
    per_token_s: float
    gpu_seconds_per_m: float  # GPU time for one million tokens (one step per token)


def kv_row_bytes(kv_dtype: str) -> int:
    """Bytes of one cached K (or V) row: 256 values in bf16 or e4m3."""
    return HEAD_DIM * (2 if kv_dtype == "bf16" else 1)


def step_counts(seq_lens: Iterable[int], kv_dtype: str, o_proj: bool = False,
                weight_bytes: int = 2) -> StepCounts:
    """Counts of one step of the layer; with ``o_proj`` the output projection (W_o, out
    read, y written) is added to the linear part. ``weight_bytes`` = 1 counts block-FP8
    projection weights (codes, plus one float32 scale per 128 x 128 block)."""
    lens = [int(n) for n in seq_lens]
    batch, positions = len(lens), sum(lens)
    row = kv_row_bytes(kv_dtype)
    qo = 2 * batch * Q_WIDTH * 2                  # q read + out written, bf16
    attn_bytes = 2 * row * positions + qo
    attn_flops = float(ATTN_FLOPS_PER_POSITION) * positions
    linear_flops = 2.0 * batch * WEIGHT_ELEMS
    # weights once; x read (bf16); q written (bf16); the appended K and V rows written
    w_bytes = WEIGHT_BYTES if weight_bytes == 2 else WEIGHT_ELEMS + 4 * (WEIGHT_ELEMS // 16384)
    linear_bytes = w_bytes + batch * HIDDEN * 2 + batch * Q_WIDTH * 2 + batch * 2 * row
    if o_proj:
        linear_flops += 2.0 * batch * O_PROJ_ELEMS
        linear_bytes += 2 * O_PROJ_ELEMS + batch * Q_WIDTH * 2 + batch * HIDDEN * 2
    return StepCounts(batch, positions, attn_flops, float(attn_bytes), linear_flops,
                      float(linear_bytes))


def step_times(c: StepCounts, hbm_gbs: float, tensor_tflops: float) -> StepTimes:
    """Roofline times of the step's two parts at the given peaks (GB/s, TFLOP/s)."""
    bw, tc = hbm_gbs * 1e9, tensor_tflops * 1e12
    a_mem, a_cmp = c.attn_bytes / bw, c.attn_flops / tc
    l_mem, l_cmp = c.linear_bytes / bw, c.linear_flops / tc
    attn, linear = max(a_mem, a_cmp), max(l_mem, l_cmp)
    step = attn + linear
    per_token = step / c.batch
    return StepTimes(attn, linear, step, "hbm" if a_mem >= a_cmp else "tensor",
                     "hbm" if l_mem >= l_cmp else "tensor", per_token, per_token * 1e6)


def layer_roofline(c: StepCounts, measured_step_s: float, hbm_gbs: float,
                   tensor_tflops: float) -> dict:
    """The modelled step against a measured one: frac = model / measured."""
    t = step_times(c, hbm_gbs, tensor_tflops)
    return {"model_us": t.step_s * 1e6, "measured_us": measured_step_s * 1e6,
            "frac": t.step_s / measured_step_s, "attention_us": t.attn_s * 1e6,
            "linear_us": t.linear_s * 1e6, "attention_bound": t.attn_bound,
            "linear_bound": t.linear_bound,
            "gpu_seconds_per_m_tokens": t.gpu_seconds_per_m}


def stack_roofline(c: StepCounts, layers: int, measured_step_s: float, hbm_gbs: float,
                   tensor_tflops: float) -> dict:
    """A stack of ``layers`` identical layer steps (each counted by ``c``) against a measured
    time for the whole stack."""
    t = step_times(c, hbm_gbs, tensor_tflops)
    model = t.step_s * layers
    return {"model_us": model * 1e6, "measured_us": measured_step_s * 1e6,
            "frac": model / measured_step_s, "layers": layers,
            "model_us_per_layer": t.step_s * 1e6,
            "measured_us_per_layer": measured_step_s * 1e6 / layers}


def main(argv: Optional[list] = None) -> None:
    """Print the model for the named workloads at the measured peaks."""
    import json
    import os
    import sys
    from decode_attention_10_b200 import workloads as W
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "MEASURED_PEAKS.json")) as f:
        peaks = json.load(f)
    names = (argv if argv is not None else sys.argv[1:]) or [w.name for w in W.WORKLOADS]
    for name in names:
        wl = W.workload(name)
        lens = W.workload_lens(wl)
        c = step_counts(lens, wl.kv_dtype)
        t = step_times(c, peaks["hbm_gbs"], peaks["bf16_tflops"])
        print(f"{wl.name}: attention {t.attn_s * 1e6:.1f} us ({t.attn_bound}), linear "
              f"{t.linear_s * 1e6:.1f} us ({t.linear_bound}), step {t.step_s * 1e6:.1f} us, "
              f"{c.batch / t.step_s:.0f} tok/s, {t.gpu_seconds_per_m:.1f} GPU-s per 1M tokens")


if __name__ == "__main__":
    main()
