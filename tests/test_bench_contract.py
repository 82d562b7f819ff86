"""The benchmark's JSON line, checked on the CPU through its reference arm (the oracle timed
on host cores), on the smallest workload: one line, the contract's keys and types, the
reference arm's own e2e and cpu_baseline objects."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_chain",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key, typ in (("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                     ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool),
                     ("scaling", str), ("dtype", str), ("data", str), ("config", dict)):
        assert isinstance(d[key], typ), (key, d[key])
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("tiny_chain")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_profile_counters_are_reported_only_while_their_sources_match(tmp_path, monkeypatch):
    """bench.py takes a kernel's DRAM traffic from its committed ncu summary only while the
    sha256 of every source the summary names still matches; a missing summary or an edited
    source gives None (the line then reports no traffic)."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "k.cuh"
    src.write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"kernel": "k", "workload": "w", "traffic_bytes_per_launch": 123,
           "sources_sha256": {"k.cuh": hashlib.sha256(src.read_bytes()).hexdigest()}}
    (tmp_path / "profiles" / "k_w.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._kernel_profile("k", "w")["traffic_bytes_per_launch"] == 123
    assert bench._kernel_profile("k", "other") is None
    src.write_text("// kernel v2\n")
    assert bench._kernel_profile("k", "w") is None


def test_committed_profiles_name_existing_sources():
    """Every committed ncu summary (json) names its kernel's sources by paths that exist,
    with a command that runs a committed entry point under ncu with --clock-control none."""
    pdir = os.path.join(ROOT, "profiles")
    recs = [f for f in os.listdir(pdir) if f.endswith(".json")]
    assert recs
    for f in recs:
        with open(os.path.join(pdir, f)) as fh:
            rec = json.load(fh)
        assert rec["sources_sha256"], f
        for rel in rec["sources_sha256"]:
            assert os.path.exists(os.path.join(ROOT, rel)), (f, rel)
        assert "--clock-control none" in rec["command"], f
        assert "tree_verify_b200.profile_case" in rec["command"], f
