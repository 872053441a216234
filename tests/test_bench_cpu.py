"""bench.py's reference arm on CPU: one JSON line with the contract's keys (the oracle, timed on the
host cores, on a bounded sample of the benchmark workload)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.timeout(600)
def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 3
    assert d["config"]["workload"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1


def test_bench_refuses_short_warmup():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode != 0


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_traffic_record_keyed_on_code_not_comments(tmp_path, monkeypatch):
    """The ncu traffic record is tied to the decode sources' code: a comment edit keeps it, a code edit
    turns the bench's traffic figure to null."""
    b = _bench_module()
    src = "// header\nint f(int x) {  // trailing\n  /* block\n comment */ return x + 1;\n}\n\n"
    assert b._code_only(src) == b._code_only(src.replace("trailing", "other words") + "// more\n")
    assert b._code_only(src) != b._code_only(src.replace("x + 1", "x + 2"))
    (tmp_path / "k.cu").write_text(src)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "DECODE_SOURCES", ("k.cu",))
    rec = {"source_hash": b.source_hash(), "dram_bytes_per_launch": 123}
    (tmp_path / "profiles" / "decode_c3_traffic.json").write_text(json.dumps(rec))
    assert b.recorded_traffic() == 123
    (tmp_path / "k.cu").write_text(src + "// a note\n")
    assert b.recorded_traffic() == 123
    (tmp_path / "k.cu").write_text(src.replace("x + 1", "x - 1"))
    assert b.recorded_traffic() is None
