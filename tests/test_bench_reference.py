"""The reference arm of bench.py keeps its output contract.

`bench.py --impl reference` times the CPU oracle on the benchmark's
workload and prints one JSON line. These runs give it a small CPU budget
(the default run takes about a minute and a half) and check the keys the
line must carry, for the decode and the prefill metric, and that a rank
other than 0 prints nothing and exits 0.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env=None):
    e = dict(os.environ, **(env or {}))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                       capture_output=True, text=True, timeout=600, env=e, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]


@pytest.mark.parametrize("extra,unit", [([], "GB/s"), (["--prefill", "1"], "TFLOP/s")])
def test_reference_line(extra, unit):
    lines = _run(["--steps", "2", "--warmup", "1", "--cpu-seconds", "0.6", *extra])
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["ms_per_step"] > 0 and d["dtype"] == "f64" and d["data"].startswith("synthetic")
    assert d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == unit and cb["cores"] >= 1
    assert cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_other_ranks_print_nothing():
    assert _run(["--gpus", "2", "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.2"],
                env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
