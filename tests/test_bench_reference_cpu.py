"""The bench's reference arm (the CPU oracle on the host cores) and its JSON line, run here on
CPU: one line with the contract's keys, a positive throughput, the oracle as cpu_baseline and an
e2e object with no host/device traffic; under a multi-rank launch only rank 0 works and prints.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    # one layer of the 8B shape keeps the host work of this check to seconds; the arm itself
    # runs all 36 layers by default
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-layers", "1"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]


def test_reference_line_keys_and_values():
    lines = _run({})
    assert len(lines) == 1
    d = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "tokens/s"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "workload" in d["config"] and d["config"]["layers"] == 1


def test_reference_other_ranks_print_nothing():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_profiling_options_parse_and_reject_bad_values():
    """The profiling options are declared, and a KV tile the attention kernel does not have is
    refused before anything runs."""
    r = subprocess.run([sys.executable, "bench.py", "--help"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0
    for opt in ("--layer-trace", "--attn-tile", "--attn-point", "--attn-m", "--probe"):
        assert opt in r.stdout, opt
    r = subprocess.run([sys.executable, "bench.py", "--workload", "attention", "--attn-tile", "32"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "invalid choice" in r.stderr
