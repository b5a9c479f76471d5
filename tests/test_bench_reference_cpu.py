"""bench.py's reference arm (the fp64 oracle on a bounded sample of the
workload) runs on CPU and prints one JSON line with the keys the benchmark
contract asks for, on the same metric and unit as the CUDA arm."""
import contextlib
import io
import json

import bench


def test_reference_arm_prints_one_complete_json_line():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference"
    assert r["metric"] == bench.METRIC and r["unit"] == "us/layer-step"
    assert r["higher_is_better"] is False and r["scaling"] == "weak" and r["vs_baseline"] is None
    assert (r["n_gpus"], r["steps"], r["warmup"]) == (1, 1, 3)
    assert r["value"] > 0 and abs(r["ms_per_step"] - r["value"] / 1e3) < 1e-3 * r["value"] / 1e3 + 1e-4
    assert r["data"] == "synthetic" and "workload" in r["config"]
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1 and cb["sample"]
    e = r["e2e"]
    assert (e["value"], e["unit"], e["h2d_bytes_per_step"], e["d2h_bytes_per_step"]) == (r["value"], r["unit"], 0, 0)
