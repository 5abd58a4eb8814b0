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
