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


def test_profile_traffic_tracks_the_kernel_sources(tmp_path, monkeypatch):
    """The roofline's DRAM traffic comes from a committed ncu summary only while the
    kernel sources still hash to the value recorded with it; otherwise it is null."""
    # a copy of the summary and of its sources: the traffic applies until a source changes
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    for rel in bench.DECODE_SOURCES:
        dst = root / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(ROOT, rel), "rb").read())
    summary = open(os.path.join(ROOT, "profiles", "ffn_decode_pg_gemma_T1.txt")).read()
    (root / "profiles" / "ffn_decode_pg_gemma_T1.txt").write_text(summary)
    monkeypatch.setattr(bench, "ROOT", str(root))
    # the summary's recorded hash is whatever the committed sources hashed to when it was taken
    recorded = [l.split(":", 1)[1].strip() for l in summary.splitlines() if l.startswith("source_sha256:")][0]
    if recorded == bench.source_hash(bench.DECODE_SOURCES):
        assert bench.profile_traffic("ffn_decode_pg_gemma_T1.txt", bench.DECODE_SOURCES) > 0
    src = root / bench.DECODE_SOURCES[0]
    src.write_bytes(src.read_bytes() + b"\n// changed\n")
    assert bench.profile_traffic("ffn_decode_pg_gemma_T1.txt", bench.DECODE_SOURCES) is None
    assert bench.profile_traffic("no_such_summary.txt", bench.DECODE_SOURCES) is None
