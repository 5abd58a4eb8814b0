"""The multi-GPU host logic of bench.py on CPU ranks (gloo, world size 2): every rank draws
its own sequences, the step time is the max over ranks, and the whole-job throughput counts
every rank's tokens. No GPU and no data-path collective are involved: sequences are
independent, so the decode step shards without any exchange."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from decode_attention_10_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.workload(1)
        # a small stand-in batch drawn the way the bench draws each rank's shard
        g = W.generate([3, 5], W.KV_BF16, seed=bench.rank_seed(wl, rank))
        xs = [torch.zeros_like(g.x) for _ in range(world)]
        dist.all_gather(xs, g.x)
        ws = [torch.zeros_like(g.w_qup[:4]) for _ in range(world)]
        dist.all_gather(ws, g.w_qup[:4])
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        out[rank] = dict(t=t, distinct=not torch.equal(xs[0].float(), xs[1].float()),
                         value=bench.whole_job_throughput(world, 2, 4, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_time_and_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        assert out[r]["t"] == 15.0          # the slower rank's time, on every rank
        assert out[r]["distinct"]           # ranks drew different sequences
        assert out[r]["value"] == pytest.approx(2 * 2 * 4 / 15e-3)


def test_single_rank_helpers_need_no_process_group():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_throughput(1, 32, 100, 10.0) == pytest.approx(320000.0)
    wl = W.workload(1)
    assert bench.rank_seed(wl, 0) == 1001 and bench.rank_seed(wl, 1) != bench.rank_seed(wl, 0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "1",
                                     "--warmup", "0"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""
