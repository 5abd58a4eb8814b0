"""Benchmark of one MFA decode step (Step-3's Multi-Matrix Factorization Attention layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME|INDEX] [--layers L]

A step is one whole decode step of the layer on one batch of synthetic inputs: hidden-state
projections (query down-projection + RMSNorm + up-projection, K/V projection + cache
append) and attention of the 64 heads over each sequence's shared K/V cache. The default
workload is batch 32 at uniform context 4096 with a bf16 KV cache.

Prints ONE JSON line (rank 0). `value` is whole-job decode throughput in tokens/s (one
token per sequence per step, summed over ranks, divided by the slowest rank's device time)
with every input already resident in HBM; `e2e` is the same metric through the public call
with the step's inputs copied from pinned host memory and its output copied back inside
the timed region. Between timed steps the inputs rotate over several device copies whose
combined footprint is far above the 126 MB L2, so no step reads the previous step's bytes
from L2. Multi-GPU runs (torchrun) shard sequences over ranks (weak scaling, no data-path
collective: the decode step of one sequence needs nothing from another).

`--layers L` times the attention side of a whole decode step instead: L layers, each the
decode step above plus the output projection 16384 -> 7168, every layer with its own weights
and cache, the whole stack one CUDA graph; its line compares the time of 61 such layers with
the pages' per-stage budgets of a 50 ms TPOT pipeline.

`--impl reference` times the float64 CPU oracle on this host's cores on a bounded sample
of the same workload (the oracle is the baseline: the pages ship no runnable code).
"""

import argparse
import itertools
import json
import math
import os
import statistics
import sys
import threading
import time
import types

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MFA decode-layer tokens/s at 4K/8K ctx; KV-stream HBM GB/s vs B200 peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "mfa_decode_b32_l4096_bf16"
L2_BYTES = 126 * 1024 * 1024
WEIGHT_BYTES = 2 * (7168 * 2048 + 2048 * 16384 + 2 * 7168 * 256)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--page-size", type=int, default=0,
                   help="keep the KV cache in shuffled pages of this many rows (a multiple of "
                        "64) behind a page table, instead of one buffer per sequence")
    p.add_argument("--weights", choices=["bf16", "fp8"], default="bf16",
                   help="projection weights in bf16, or block-FP8 (e4m3 codes, one float32 "
                        "scale per 128 x 128 block; the layer uses bf16(code * scale))")
    p.add_argument("--page-order", choices=["shuffled", "sequential"], default="shuffled",
                   help="with --page-size: pages handed out in random or in sequence order")
    p.add_argument("--passes", type=int, default=0,
                   help="timed passes of --steps steps each (default: enough for about "
                        "0.25 s of timed work, at least 5); the value is the median pass")
    p.add_argument("--no-extra-workloads", action="store_true",
                   help="time the chosen workload only (by default a single-GPU run of the "
                        "default workload also times the 8K, FP8 and ragged workloads)")
    p.add_argument("--layers", type=int, default=0,
                   help="time the attention side of a whole decode step instead: this many "
                        "layers, each the MFA decode step plus its output projection")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(wl, rank: int) -> int:
    """Each rank draws its own sequences (weak scaling: sequences are sharded, weights are
    replicated and drawn identically on every rank)."""
    return 1000 + wl.index + 7919 * rank


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time: every multi-GPU number is the max over ranks."""
    if world <= 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(world: int, batch_per_rank: int, steps: int, t_ms: float) -> float:
    """Tokens/s of the whole job: one token per sequence per step on every rank."""
    return world * batch_per_rank * steps / (t_ms / 1e3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s for a kernel timed alone (burst), measured, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


# ---------------------------------------------------------------------------------------
# clocks during the timed region (NVML in a thread; read-only queries)
# ---------------------------------------------------------------------------------------


class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int):
        self.ok = False
        self.samples = []
        self.reasons = 0
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - NVML missing
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------------------


def oracle_sample_throughput(inp, n_seq: int):
    """Time the oracle's whole decode step for the first n_seq sequences; tokens/s."""
    import numpy as np
    from oracle import codecs
    from oracle import mfa as omfa

    def f64(t):
        import torch
        return codecs.bf16_decode(t.contiguous().view(torch.int16).numpy().view(np.uint16))

    def codes(t):
        import torch
        t = t.contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.view(torch.uint8).numpy()

    od = omfa.KV_BF16 if inp.kv_dtype == "bf16" else omfa.KV_FP8
    w = [f64(inp.w_qdown), f64(inp.gamma), f64(inp.w_qup), f64(inp.w_k), f64(inp.w_v)]
    x = f64(inp.x)[:n_seq]
    kc = [codes(inp.k_cache[b]) for b in range(n_seq)]
    vc = [codes(inp.v_cache[b]) for b in range(n_seq)]
    lens = inp.seq_lens.tolist()[:n_seq]
    t0 = time.perf_counter()
    omfa.decode_layer(x, *w, kc, vc, lens, od, inp.k_scale, inp.v_scale)
    dt = time.perf_counter() - t0
    return n_seq / dt, dt


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------------------


def attention_bytes(inp) -> int:
    """Algorithmic HBM bytes of one attention launch: every attended K and V row once, q
    read once and out written once per sequence."""
    row = 256 * (2 if inp.kv_dtype == "bf16" else 1)
    kv = 2 * row * int(inp.seq_lens.sum())
    qo = 2 * inp.batch * 64 * 256 * 2
    return kv + qo


def kv_bytes(inp) -> int:
    row = 256 * (2 if inp.kv_dtype == "bf16" else 1)
    return 2 * row * int(inp.seq_lens.sum())


def timed_passes(run_pass, passes, world, dev):
    """Run `passes` timed passes. Each pass is bracketed by a barrier and a synchronize on
    both sides; run_pass records its own CUDA events on the stream(s) it launches on and
    returns the elapsed device time (ms). Per pass, the slowest rank's time."""
    import torch
    out = []
    for _ in range(passes):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ms = run_pass()
        if world > 1:
            torch.distributed.barrier()
        out.append(max_over_ranks(ms, world, dev))
    return out


def pick_passes(args, pass_ms_estimate: float) -> int:
    """Passes of K steps: --passes if given, else enough for about 0.25 s of timed work (so
    the clock samples cover a steady state), at least 5 and at most 300."""
    if args.passes > 0:
        return args.passes
    return int(min(300, max(5, math.ceil(250.0 / max(pass_ms_estimate, 1e-3)))))


def pass_summary(times):
    return {"passes": len(times), "median_ms": statistics.median(times), "min_ms": min(times),
            "max_ms": max(times)}


def run_ours(args, wl, rank, world, local, headline=True):
    """Measure one workload: the whole decode step (CUDA-graph replay, inputs resident in
    HBM), the attention call alone, and (headline only) the end-to-end public call with
    host copies and the CPU oracle baseline."""
    import torch
    from decode_attention_10_b200 import build, mfa
    from decode_attention_10_b200 import workloads as W
    from decode_attention_10_b200.cost_model import layer_roofline, step_counts

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp = W.generate_workload(wl, seed=rank_seed(wl, rank))
    bsz = inp.batch
    step_bytes = (WEIGHT_BYTES // (2 if args.weights == "fp8" else 1)) + kv_bytes(inp)
    copies = max(2, math.ceil(3 * L2_BYTES / step_bytes))
    K = args.steps

    class Copy:
        pass

    sets = []
    for _ in range(copies):
        c = Copy()
        c.x = inp.x.to(dev)
        c.w = [t.to(dev) for t in (inp.w_qdown, inp.gamma, inp.w_qup, inp.w_k, inp.w_v)]
        if args.weights == "fp8":
            c.w = [c.w[1] if i == 1 else mfa.BlockFP8Weight(*W.quantize_w8(t))
                   for i, t in enumerate(c.w)]
        if inp.k_buffer is not None:
            kb, vb = inp.k_buffer.to(dev), inp.v_buffer.to(dev)
            c.k, c.v = [kb[b] for b in range(bsz)], [vb[b] for b in range(bsz)]
            c.keep = (kb, vb)
        else:
            c.k = [t.to(dev) for t in inp.k_cache]
            c.v = [t.to(dev) for t in inp.v_cache]
        if args.page_size:
            kp, vp, pt, npages = W.to_paged(c.k, c.v, args.page_size, seed=len(sets),
                                            shuffle=args.page_order == "shuffled")
            c.keep = (kp, vp, pt)
            c.k = c.v = None
            c.cache = mfa.PagedKVCache(kp, vp, pt, npages, inp.k_scale, inp.v_scale)
        else:
            c.cache = mfa.KVCache(c.k, c.v, inp.k_scale, inp.v_scale)
        c.q = torch.empty(bsz, 64, 256, dtype=torch.bfloat16, device=dev)
        c.out = torch.empty(bsz, 64, 256, dtype=torch.bfloat16, device=dev)
        sets.append(c)
    lens = inp.seq_lens.to(dev)
    ws = mfa.Workspace(bsz, dev)
    for c in sets:
        c.step = mfa.DecodeStep(c.x, *c.w, c.cache, lens, c.q, c.out, ws)

    for i in range(args.warmup):
        sets[i % copies].step()
    torch.cuda.synchronize()
    if mfa.get_error(ws) != 0:
        raise RuntimeError("device error flag set during warm-up")
    if not torch.isfinite(sets[0].out.float()).all():
        raise RuntimeError("non-finite output")

    # host cost of one call of the public API: the median time to enqueue one call into an
    # idle stream (no device work waited for, no queue back-pressure); the same for a replay
    # of the step captured by the library (mfa_decode_layer_graph); and the mean over 50
    # calls back to back, whose later calls can wait for room in the launch queue
    def enqueue_us(call, reps=200):
        times = []
        for _ in range(reps):
            torch.cuda.synchronize()
            h0 = time.perf_counter()
            call()
            times.append((time.perf_counter() - h0) * 1e6)
        torch.cuda.synchronize()
        return statistics.median(times)

    host_us = enqueue_us(sets[0].step)
    captured = mfa.StepGraph(sets[0].x, *sets[0].w, sets[0].cache, lens, sets[0].q,
                             sets[0].out, ws)
    captured()
    host_us_graph = enqueue_us(captured)
    captured.close()
    torch.cuda.synchronize()
    n_host = 50
    h0 = time.perf_counter()
    for i in range(n_host):
        sets[i % copies].step()
    host_us_queued = (time.perf_counter() - h0) / n_host * 1e6
    torch.cuda.synchronize()

    # The K steps of a pass captured once as one CUDA graph over the rotating copies (the
    # kernels, their arguments and tensor maps are recorded; replay re-runs exactly those
    # launches). Inside it each step's first kernel is a programmatic dependent of the previous
    # step's last, as consecutive layers are on a serving stream: it streams its first weight
    # stages while the previous combine runs and reads x only once that step has completed.
    # Each copy's step is also captured alone, for the isolated-step figure.
    graphs = []
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for c in sets:
            g = torch.cuda.CUDAGraph()
            c.gstep = mfa.DecodeStep(c.x, *c.w, c.cache, lens, c.q, c.out, ws, stream=side)
            with torch.cuda.graph(g, stream=side):
                c.gstep()
            graphs.append(g)
        pass_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pass_graph, stream=side):
            for i in range(K):
                sets[i % copies].gstep()
    torch.cuda.current_stream().wait_stream(side)
    for i in range(max(args.warmup, 2)):
        graphs[i % copies].replay()
    pass_graph.replay()
    torch.cuda.synchronize()

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def graph_pass():
        ev[0].record()
        pass_graph.replay()
        ev[1].record()
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1])

    def isolated_pass():
        ev[0].record()
        for i in range(K):
            graphs[i % copies].replay()
        ev[1].record()
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1])

    def attn_pass():
        ev[0].record()
        for i in range(K):
            c = sets[i % copies]
            mfa.decode_attn(c.q, c.cache, lens, out=c.out, ws=ws)
        ev[1].record()
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1])

    # 1) the timed region: passes of exactly K whole decode steps (graph replays); the
    #    value is the median pass, the clocks are sampled across all passes
    passes = pick_passes(args, max_over_ranks(graph_pass(), world, dev))  # same on every rank
    with ClockSampler(local) as clk:
        step_times = timed_passes(graph_pass, passes, world, dev)
    t_ms = statistics.median(step_times)
    ms_per_step = t_ms / K
    value = whole_job_throughput(world, bsz, K, t_ms)

    # the same K steps as K separate graph replays: no step overlaps its neighbours
    isolated_pass()
    iso_times = timed_passes(isolated_pass, max(5, passes // 2), world, dev)

    # 2) the attention launch alone: K calls back to back over the rotating copies, CUDA
    #    events on the launching stream around each pass (inter-launch gaps included)
    attn_pass()
    attn_times = timed_passes(attn_pass, max(5, passes // 2), world, dev)
    attn_ms = statistics.median(attn_times) / K

    peak, peak_kind = measured_peaks()
    a_bytes = attention_bytes(inp)
    achieved = a_bytes / (attn_ms / 1e3) / 1e9
    traffic = None if args.page_size else profiled_traffic(wl.name)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if inp.kv_dtype == "bf16" else "bf16+fp8kv", "data": "synthetic",
        "config": {"workload": wl.name, "batch_per_gpu": bsz, "global_batch": bsz * world,
                   "context": wl.context, "kv_dtype": inp.kv_dtype,
                   "weights": ("block-fp8 e4m3, 128 x 128 blocks" if args.weights == "fp8"
                               else "bf16"),
                   "kv_layout": (f"paged, {args.page_size} rows per page, {args.page_order}"
                                 if args.page_size else "one buffer per sequence"),
                   "heads": 64, "head_dim": 256, "hidden": 7168, "q_rank": 2048,
                   "l2": f"inputs rotate over {copies} device copies "
                         f"({step_bytes / 1e6:.0f} MB each, > 126 MB L2)",
                   "parallelism": f"dp{world} (sequences sharded, weights replicated)"},
        "kv_gbs": kv_bytes(inp) / (attn_ms / 1e3) / 1e9,
        "attn_ms": attn_ms,
        "roofline": {"kernel": "mfa_decode_attn: split-K attention (split plan built on chip) "
                               "+ combine (2 launches, timed together)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "bytes_per_launch": a_bytes, "traffic": traffic},
        # the whole step against its roofline: max(flops/TC, bytes/HBM) for the attention plus
        # the same for the linear projections (the pages' cost framing), at the measured peaks
        "layer_roofline": layer_roofline(step_counts(inp.seq_lens.tolist(), inp.kv_dtype,
                                                     weight_bytes=1 if args.weights == "fp8"
                                                     else 2),
                                         ms_per_step / 1e3, peak, measured_tensor_peak()),
        "clocks": clk.summary(),
        "step_passes": pass_summary(step_times),
        "ms_per_step_isolated": statistics.median(iso_times) / K,
        "attn_passes": pass_summary(attn_times),
        "gpu_launches": (LAUNCHES_PER_LAYER if args.weights == "bf16" else LAUNCHES_PER_LAYER_W8) * K,
        "host_us_per_call": host_us,
        "host_us_per_call_graph": host_us_graph,
        "host_us_per_call_queued": host_us_queued,
    }
    if not headline:
        return result

    # 3) end to end through the public call with host buffers: every step copies its x and
    #    seq_lens in from pinned host memory (one copy: x and seq_lens are adjacent in one
    #    device buffer) and reads its output back, inputs on one copy stream and outputs on
    #    another. Each step's output goes back as soon as that step is done (an event record
    #    on the compute stream, which does not hold the next step back); inputs go in by
    #    groups of steps (1, then 4, then E2E_GROUP at a time, as the layers of a token step
    #    run between its copies), and the compute stream waits for a group's inputs only
    #    before the group, so inside a group each step chains to the previous one as in the
    #    device-timed passes. Step i uses buffer i % n_buf; events order every reuse.
    x_bytes = bsz * 7168 * 2
    in_bytes = x_bytes + 4 * bsz
    n_buf = 2 * E2E_GROUP
    comp = torch.cuda.Stream(dev)
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    bufs = []
    for j in range(n_buf):
        buf = torch.empty(in_bytes + 256, dtype=torch.uint8, device=dev)
        xe = buf[:x_bytes].view(torch.bfloat16).view(bsz, 7168)
        lens_e = buf[x_bytes:in_bytes].view(torch.int32)
        out_e = torch.empty(bsz, 64, 256, dtype=torch.bfloat16, device=dev)
        hb = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
        hb[:x_bytes].view(torch.bfloat16).view(bsz, 7168).copy_(inp.x)
        hb[x_bytes:].view(torch.int32).copy_(inp.seq_lens)
        bufs.append(types.SimpleNamespace(
            in_dev=buf[:in_bytes], host_in=hb, out=out_e,
            out_host=torch.empty(bsz, 64, 256, dtype=torch.bfloat16).pin_memory(),
            # step i runs weight set i % copies on buffer i % n_buf: one bound call per set
            step={k: mfa.DecodeStep(xe, *sets[k].w, sets[k].cache, lens_e, sets[k].q, out_e,
                                    ws, stream=comp) for k in range(copies)},
            c_evt=torch.cuda.Event(),  # its step computed (inputs consumed)
            d_evt=torch.cuda.Event()))  # its output read back
    groups = e2e_groups(K, E2E_GROUP)
    # two consecutive groups never hold more than n_buf steps, so the copies of group g + 1,
    # enqueued after group g's first call, wait only for steps of groups before g, whose
    # events are recorded (and not yet recorded again by group g, whose buffers differ)
    assert all(len(a) + len(b) <= n_buf for a, b in zip(groups, groups[1:]))
    h_evt = [torch.cuda.Event() for _ in range(2)]  # inputs of group g in (by g % 2)
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def h2d(gi):  # on h2d_s: group gi's inputs, each once its buffer's previous step is done
        for i in groups[gi]:
            b = bufs[i % n_buf]
            if i >= n_buf:
                h2d_s.wait_event(b.c_evt)
            b.in_dev.copy_(b.host_in, non_blocking=True)
        h_evt[gi % 2].record(h2d_s)

    def e2e_pass():
        comp.wait_stream(torch.cuda.current_stream())
        h2d_s.wait_stream(comp)
        d2h_s.wait_stream(comp)
        with torch.cuda.stream(h2d_s):
            e2e_ev[0].record(h2d_s)
            h2d(0)
        for gi, grp in enumerate(groups):
            comp.wait_event(h_evt[gi % 2])
            if grp[-1] >= n_buf:  # the group's buffers' previous outputs have been read back
                comp.wait_event(bufs[grp[-1] % n_buf].d_evt)
            for i in grp:
                b = bufs[i % n_buf]
                b.step[i % copies]()
                b.c_evt.record(comp)
                if i == grp[0] and gi + 1 < len(groups):
                    # the next group's inputs go in while this group computes: enqueued once
                    # the group's first call is (so the GPU does not wait for the host to
                    # issue them), and before any of the group's read-backs, which would
                    # otherwise hold them back in the copy queue
                    with torch.cuda.stream(h2d_s):
                        h2d(gi + 1)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(b.c_evt)
                    b.out_host.copy_(b.out, non_blocking=True)
                    b.d_evt.record(d2h_s)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_stream(comp)
            d2h_s.wait_stream(h2d_s)
            e2e_ev[1].record(d2h_s)
        torch.cuda.synchronize()
        return e2e_ev[0].elapsed_time(e2e_ev[1])

    e2e_pass()
    e2e_times = timed_passes(e2e_pass, max(5, min(passes, 20)), world, dev)
    # every step computes the same inputs on its weight set: what each buffer read back last
    # must be that set's output of the device-timed steps
    for i in range(max(0, K - n_buf), K):
        b = bufs[i % n_buf]
        if not torch.equal(b.out_host, sets[i % copies].out.cpu()):
            raise RuntimeError("e2e: an output read back differs from the step's result")
    t_e2e = statistics.median(e2e_times)
    result["e2e"] = {"value": whole_job_throughput(world, bsz, K, t_e2e), "unit": UNIT,
                     "h2d_bytes_per_step": in_bytes,
                     "d2h_bytes_per_step": bsz * 64 * 256 * 2,
                     "group": E2E_GROUP, "passes": pass_summary(e2e_times)}
    result["timing"] = ("value: median of passes of one CUDA-graph replay of K whole steps "
                        "(each step chained to the previous one by programmatic dependent "
                        "launch); ms_per_step_isolated: the same steps as K separate graph "
                        "replays; "
                        "e2e: median of passes of K public-API calls, each step's inputs "
                        "copied in (by groups of 1, 4, then E2E_GROUP steps) and its output "
                        "copied back, on two copy streams that overlap the compute; "
                        "attn: median of passes of "
                        "K back-to-back mfa_decode_attn calls")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # whole decode steps of the first n_seq sequences, repeated until about 10 s of CPU
        # work (at most 20 repetitions)
        n_seq = min(bsz, 32)
        tokens, total, reps = 0, 0.0, 0
        while total < 10.0 and reps < 20:
            _, dt = oracle_sample_throughput(inp, n_seq)
            tokens, total, reps = tokens + n_seq, total + dt, reps + 1
        result["cpu_baseline"] = {"value": tokens / total, "unit": UNIT, "cores": cpu_cores(),
                                  "kind": "oracle",
                                  "sample": f"{reps} whole decode steps of {n_seq} of the "
                                            f"{bsz} sequences (float64 numpy), {total:.1f} s"}
    return result


def run_extra_workloads(args, rank, world, local):
    """The other full-size workloads, measured the same way as the headline (whole step and
    attention call; no host copies, no CPU baseline), each with its own clocks."""
    import gc

    import torch
    from decode_attention_10_b200 import workloads as W
    out = {}
    gc.collect()
    torch.cuda.empty_cache()
    for name in EXTRA_WORKLOADS:
        r = run_ours(args, W.workload(name), rank, world, local, headline=False)
        out[name] = {k: r[k] for k in ("value", "ms_per_step", "ms_per_step_isolated",
                                       "attn_ms", "kv_gbs", "roofline",
                                       "layer_roofline", "clocks", "step_passes",
                                       "attn_passes")}
        out[name]["config"] = {k: r["config"][k] for k in ("batch_per_gpu", "context",
                                                           "kv_dtype", "kv_layout")}
        gc.collect()
        torch.cuda.empty_cache()
    return out


def e2e_groups(steps: int, largest: int):
    """The end-to-end passes' groups of consecutive steps: 1, then 4, then `largest` at a time
    (the first group small so that the first call waits for one input copy only), the last
    group what is left. Returns ranges that cover 0 .. steps - 1 in order."""
    groups, g0 = [], 0
    for size in itertools.chain((1, 4), itertools.repeat(largest)):
        if g0 >= steps:
            break
        groups.append(range(g0, min(g0 + min(size, largest), steps)))
        g0 = groups[-1].stop
    return groups


# Largest group of steps whose inputs the end-to-end passes copy in together: the calls of a
# group run back to back on the compute stream (a few layers of one token step of a model).
E2E_GROUP = 8


# The workloads timed after the headline in a default run: the 8K point of the metric, the
# FP8 cache at 4K, and the ragged long-context batch.
EXTRA_WORKLOADS = ("mfa_decode_b64_l8192_bf16", "mfa_decode_b128_l4096_fp8",
                   "mfa_decode_b16_ragged64k_bf16")


LAUNCHES_PER_LAYER = 5  # x-projection, split-K finish (+RMSNorm, append, split plan), q_up,
#                         attention, split combine
LAUNCHES_PER_LAYER_W8 = 6  # FP8 weights: the same plus the quantization of x


# The pages' per-stage budgets of a 50 ms TPOT pipeline, summed over the 61 layers (bud-325
# "Key claims": 16.6 ms per stage with 3 stages, 12.5 ms with 4).
STAGE_BUDGET_MS = {"3-stage": 16.6, "4-stage": 12.5}
MODEL_LAYERS = 61


def run_stack(args, wl, rank, world, local):
    """The attention side of one decode step: ``args.layers`` layers on one stream, each the
    MFA decode step of the workload's batch and its output projection 16384 -> 7168, layer
    l + 1 taking layer l's projection as its hidden input (the FFN between them runs on
    other GPUs under Attention-FFN Disaggregation and is not part of this path). Every layer
    has its own weights and KV cache in HBM; the whole stack is one CUDA graph."""
    import torch
    from decode_attention_10_b200 import build, mfa
    from decode_attention_10_b200 import workloads as W
    from decode_attention_10_b200.cost_model import stack_roofline, step_counts

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    seed = rank_seed(wl, rank)
    lens_list = W.workload_lens(wl, seed=seed)
    bsz = len(lens_list)
    nl = args.layers
    layers = [W.generate_layer_on_device(lens_list, wl.kv_dtype, seed * 1000 + l, dev,
                                         contiguous=wl.contiguous) for l in range(nl)]
    g = torch.Generator(device=dev).manual_seed(seed)
    x0 = torch.randn(bsz, 7168, generator=g, device=dev).to(torch.bfloat16)
    lens = torch.tensor(lens_list, dtype=torch.int32, device=dev)
    ws = mfa.Workspace(bsz, dev)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    x = x0
    for lay in layers:
        lay["cache"] = mfa.KVCache(lay["k_cache"], lay["v_cache"], lay["k_scale"],
                                   lay["v_scale"])
        lay["x"] = x
        lay["q"] = torch.empty(bsz, 64, 256, dtype=torch.bfloat16, device=dev)
        lay["out"] = torch.empty(bsz, 64, 256, dtype=torch.bfloat16, device=dev)
        lay["y"] = torch.empty(bsz, 7168, dtype=torch.bfloat16, device=dev)
        lay["step"] = mfa.DecodeStep(x, lay["w_qdown"], lay["gamma"], lay["w_qup"], lay["w_k"],
                                     lay["w_v"], lay["cache"], lens, lay["q"], lay["out"], ws,
                                     stream=side)
        x = lay["y"]

    def stack():
        for lay in layers:
            lay["step"]()
            mfa.o_proj(lay["out"], lay["w_o"], y=lay["y"], ws=ws, stream=side)

    with torch.cuda.stream(side):
        stack()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            stack()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(max(args.warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()
    if mfa.get_error(ws) != 0:
        raise RuntimeError("device error flag set during warm-up")
    if not torch.isfinite(layers[-1]["y"].float()).all():
        raise RuntimeError("non-finite output")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record()
        for _ in range(args.steps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_per_step = t_ms / args.steps
    peak, _ = measured_peaks()
    counts = step_counts(lens_list, wl.kv_dtype, o_proj=True)
    per_layer_ms = ms_per_step / nl
    return {
        "metric": "MFA attention-side decode tokens/s (layers x [decode step + output "
                  "projection])",
        "value": whole_job_throughput(world, bsz, args.steps, t_ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.kv_dtype == "bf16" else "bf16+fp8kv", "data": "synthetic",
        "config": {"workload": wl.name, "layers": nl, "batch_per_gpu": bsz,
                   "global_batch": bsz * world, "context": wl.context,
                   "kv_dtype": wl.kv_dtype, "o_proj": "16384 -> 7168",
                   "l2": "every layer has its own weights and KV cache "
                         f"({(counts.linear_bytes + counts.attn_bytes) / 1e6:.0f} MB per "
                         "layer, > 126 MB L2)",
                   "parallelism": f"dp{world} (sequences sharded, weights replicated)"},
        "ms_per_layer": per_layer_ms,
        "stage_ms_61_layers": per_layer_ms * MODEL_LAYERS,
        "stage_budget_ms": STAGE_BUDGET_MS,
        "within_budget": {k: per_layer_ms * MODEL_LAYERS <= v
                          for k, v in STAGE_BUDGET_MS.items()},
        "stack_roofline": stack_roofline(counts, nl, ms_per_step / 1e3, peak,
                                         measured_tensor_peak()),
        "clocks": clk.summary(),
        "gpu_launches": 7 * nl * args.steps,
        "timing": "CUDA-graph replay of the whole stack; CUDA events on the launching "
                  "stream",
    }


def profiled_traffic(workload_name):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on
    the current attention source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            d = json.load(f)
        import hashlib
        h = hashlib.sha256()
        for name in d.get("sources", []):
            with open(os.path.join(ROOT, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != d.get("source_sha256"):
            return None
        entry = d.get("per_launch", {}).get(workload_name)
        return None if entry is None else float(entry)
    except Exception:
        return None


def run_reference(args, wl, rank, world):
    """The oracle on host cores, on the same workload: each step is one whole decode step
    of a bounded sample of the batch."""
    from decode_attention_10_b200 import workloads as W
    inp = W.generate_workload(wl)
    n_seq = min(inp.batch, 2)
    for _ in range(args.warmup):
        oracle_sample_throughput(inp, n_seq)
    times = []
    for _ in range(args.steps):
        _, dt = oracle_sample_throughput(inp, n_seq)
        times.append(dt)
    total = sum(times)
    value = n_seq * len(times) / total
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch_per_gpu": inp.batch, "context": wl.context,
                   "kv_dtype": inp.kv_dtype, "sample_sequences_per_step": n_seq},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"{n_seq} of {inp.batch} sequences per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_env()
    from decode_attention_10_b200 import workloads as W
    try:
        wl = W.workload(int(args.workload))
    except ValueError:
        wl = W.workload(args.workload)
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, wl, rank, world)), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.layers > 0:
            res = run_stack(args, wl, rank, world, local)
        else:
            res = run_ours(args, wl, rank, world, local)
            if (world == 1 and wl.name == DEFAULT_WORKLOAD and not args.no_extra_workloads
                    and not args.page_size and args.weights == "bf16"):
                res["workloads"] = run_extra_workloads(args, rank, world, local)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
