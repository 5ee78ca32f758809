"""The bench's reference arm (the fp64 oracle on the host cores) prints the JSON
line the benchmark contract asks for, on the same workload as the GPU arm."""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line(capsys, monkeypatch):
    monkeypatch.delenv("RANK", raising=False)
    bench.run_reference(argparse.Namespace(steps=2, warmup=1, gpus=1))
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == bench.DECODE_WORKLOAD
    assert (d["config"]["d_model"], d["config"]["r"], d["config"]["d_ff"], d["config"]["k"]) == \
        (bench.D_MODEL, bench.R, bench.D_FF, bench.K)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
