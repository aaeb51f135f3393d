"""The bench's reference arm on the CPU: `bench.py --impl reference` times the
float64 oracle on the host cores and prints one JSON line with the contract's
keys (no GPU is needed, so this runs everywhere)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "1",
           "--ref-sample-tokens", "32"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    # value = tokens of the timed steps / their time
    assert abs(d["value"] - 2 * 32 / (2 * d["ms_per_step"] / 1000)) <= 1e-6 * d["value"]
    assert d["config"]["workload"] == "qwen3_0.6b_block_T65536"
    assert d["config"]["sample_tokens"] == 32
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "32 tokens" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
