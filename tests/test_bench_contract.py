"""bench.py's JSON line, checked on the CPU through its reference arm (the float64 oracle on
the host cores), which needs no GPU: the keys and units the round driver reads, the reference
arm's own cpu_baseline and e2e objects, and the rejection of a warm-up below three steps."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=240):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=timeout)


def _last_json(stdout: str) -> dict:
    lines = [l for l in stdout.splitlines() if l.startswith("{")]
    assert lines, stdout
    return json.loads(lines[-1])


@pytest.mark.parametrize("extra,metric_word,unit", [
    (["--workload", "decode_tiny_f32"], "decode", "tokens/s"),
    (["--workload", "prefill_b4_t4k", "--batch", "1", "--seq-len", "64"], "prefill", "tokens/s"),
])
def test_reference_arm_line(extra, metric_word, unit):
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", *extra)
    assert r.returncode == 0, r.stderr[-2000:]
    d = _last_json(r.stdout)
    assert d["impl"] == "reference"
    assert metric_word in d["metric"]
    assert d["unit"] == unit and d["value"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["scaling"] in ("weak", "strong") and d["data"] and d["dtype"]
    assert isinstance(d["config"], dict) and d["config"]["workload"] == extra[1]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == pytest.approx(d["value"]) and cb["unit"] == d["unit"]
    e2e = d["e2e"]
    assert e2e["unit"] == d["unit"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_rejected():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "2", "--workload", "decode_tiny_f32")
    assert r.returncode != 0
    assert "warmup" in r.stderr
