"""The measurement harness on the CPU: the reference arm (the oracle timed on
the host cores) prints one JSON line with every key the bench line carries,
the timing rules are enforced on the command line, and the committed DRAM
traffic figure is used only while the kernel sources it was taken from are
unchanged."""
import json
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def run_bench(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_complete_line(oracle_mod):
    res = run_bench("--impl", "reference", "--steps", "1", "--warmup", "3",
                    "--ref-step-seconds", "0.2")
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["warmup"] == 3 and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] and d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_fewer_than_three_warmup_steps_are_refused():
    res = run_bench("--impl", "reference", "--steps", "1", "--warmup", "2", timeout=120)
    assert res.returncode != 0 and "warmup" in res.stderr


def test_traffic_figure_is_dropped_when_its_sources_change(tmp_path, monkeypatch):
    # A tree with one kernel source and a traffic record carrying that
    # source's hash: the record is used while the source is unchanged and
    # dropped (None) once one byte of it changes.
    import hashlib
    import json

    import bench
    root = tmp_path / "tree"
    (root / "profiles").mkdir(parents=True)
    src = root / "k.cu"
    src.write_bytes(b"__global__ void k() {}\n")
    rec = {"k": {"bytes_per_launch": 123, "sources": ["k.cu"],
                 "sources_sha256": hashlib.sha256(src.read_bytes()).hexdigest()}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(root))
    t = bench.profile_traffic("k")
    assert t is not None and t["bytes_per_launch"] == 123
    src.write_bytes(src.read_bytes() + b"\n")
    assert bench.profile_traffic("k") is None
    assert bench.profile_traffic("no_such_kernel") is None
