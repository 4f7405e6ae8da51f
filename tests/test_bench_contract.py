"""bench.py's reference arm (the CPU oracle) prints the JSON line the bench
contract asks for.  Runs on CPU; the GPU arm is exercised on a GPU machine."""
import contextlib
import io
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.slow
def test_reference_arm_json_line():
    sys.path.insert(0, ROOT)
    import bench

    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--ref-fraction", "0.002"])
    assert rc == 0
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    with open(os.path.join(ROOT, "BASELINE.json")) as fh:
        metric = json.load(fh)["metric"]
    assert line["impl"] == "reference"
    assert line["metric"] == metric
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["steps"] == 1 and line["warmup"] == 0 and line["n_gpus"] == 1
    assert line["data"] == "synthetic" and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["config"]["workload"].startswith("SwiGLU MLP block")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
