"""The benchmark's JSON line, checked on the CPU through its reference arm.

`bench.py --impl reference` times the oracle on the host cores and prints the
same line layout as the CUDA arm (plus `impl`, `requested`, `cpu_baseline` and
`e2e` describing itself); the CUDA arm builds its `config` object with the same
function.  This runs the arm on the tiny workload and checks the keys, types
and the relations the line's readers rely on.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _reference_line(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          *extra], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line_follows_the_contract():
    d = _reference_line("--steps", "2", "--warmup", "1")
    for key, kind in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                      ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                      ("dtype", str), ("data", str), ("config", dict), ("impl", str), ("cpu_baseline", dict),
                      ("e2e", dict)]:
        assert isinstance(d[key], kind), (key, d[key])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # one full step is timed and reported as such; the request is echoed
    assert d["steps"] == 1 and d["warmup"] == 0
    assert d["requested"] == {"steps": 2, "warmup": 1}
    # tokens/s = S (R - 1) per step, within the rounding of the printed ms_per_step (0.1 ms here)
    ms = d["ms_per_step"]
    assert 256 * 3 / ((ms + 0.05) * 1e-3) - 1.0 <= d["value"] <= 256 * 3 / ((ms - 0.05) * 1e-3) + 1.0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cfg = d["config"]
    assert set(cfg) == {"workload", "l2", "parallelism", "active_tokens", "attention_pairs"}
    assert cfg["workload"].startswith("tiny:")
    assert cfg["l2"].startswith("inputs smaller than L2")
    assert set(cfg["active_tokens"]) == {"loop2", "loop3", "loop4"}
    # the planted schedule: 75 % / 40 % / 20 % of 256 tokens, rounded half up
    assert cfg["active_tokens"] == {"loop2": 192, "loop3": 102, "loop4": 51}
    assert all(v > 0 for v in cfg["attention_pairs"].values())
