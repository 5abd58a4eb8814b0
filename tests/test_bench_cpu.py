"""bench.py's CPU-side contract: the reference arm (the float64 oracle timed on the host's
cores) prints one JSON line with the keys the driver reads."""

import json

import bench


def test_reference_arm_prints_one_json_line(monkeypatch, capsys):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--workload",
                                     "mfa_decode_b1_l128_bf16", "--steps", "1", "--warmup", "0"])
    assert bench.main() == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e", "impl"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["workload"] == "mfa_decode_b1_l128_bf16"
    assert d["metric"] == bench.METRIC


def test_attention_bytes_are_the_algorithmic_count():
    from decode_attention_10_b200 import workloads as W
    inp = W.generate([100, 300], W.KV_BF16, seed=1)
    # K and V rows once (2 x 512 B per position), q read and out written (2 x 32 KB per seq)
    assert bench.attention_bytes(inp) == 2 * 512 * 400 + 2 * 2 * 64 * 256 * 2
    inp8 = W.generate([100, 300], W.KV_FP8, seed=1)
    assert bench.kv_bytes(inp8) == 2 * 256 * 400


def test_paged_layout_holds_every_sequence_row_in_its_listed_pages():
    import torch

    from decode_attention_10_b200 import workloads as W
    for dtype, page in (("bf16", 128), ("fp8_e4m3", 64), ("bf16", 192)):
        inp = W.generate([5, 130, 300], dtype, seed=1, capacity=[64, 200, 300])
        kp, vp, pt, need = W.to_paged(inp.k_cache, inp.v_cache, page, seed=3, spare_pages=2)
        assert kp.shape == (sum(need) + 2, page, 256) and kp.dtype == inp.k_cache[0].dtype
        assert need == [-(-c // page) for c in (64, 200, 300)]
        used = pt[0, :need[0]].tolist() + pt[1, :need[1]].tolist() + pt[2, :need[2]].tolist()
        assert len(set(used)) == len(used)  # no page shared
        for pool, cache in ((kp, inp.k_cache), (vp, inp.v_cache)):
            for b, t in enumerate(cache):
                raw = pool.view(torch.uint8) if t.element_size() == 1 else pool.view(torch.int16)
                rows = torch.cat([raw[int(pt[b, p])] for p in range(need[b])])[:t.shape[0]]
                want = t.view(torch.uint8) if t.element_size() == 1 else t.view(torch.int16)
                assert torch.equal(rows, want)


def test_e2e_groups_cover_the_steps_in_order_within_the_buffer_ring():
    import bench
    for largest in (1, 4, 8):
        for steps in range(1, 60):
            groups = bench.e2e_groups(steps, largest)
            flat = [i for g in groups for i in g]
            assert flat == list(range(steps))
            assert len(groups[0]) == 1 and all(1 <= len(g) <= largest for g in groups)
            # the e2e loop reuses a ring of 2 * largest buffers: two consecutive groups fit it
            assert all(len(a) + len(b) <= 2 * largest for a, b in zip(groups, groups[1:]))
