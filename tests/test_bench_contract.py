"""bench.py's reference arm (the float64 oracle on the host) keeps the JSON
contract the driver reads: one line with the metric, value, unit, the
reference marker, the CPU baseline and an end-to-end entry.  CPU only."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["steps"] == 2                                       # every requested step is timed
    assert d["cpu_baseline"]["nproc"] >= d["cpu_baseline"]["cores"]
    assert int(d["cpu_baseline"]["affinity"], 16) > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_profiled_fields_follow_the_source_hash(tmp_path):
    """A committed ncu summary is used only while the kernel sources still hash
    to the value recorded with it."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "csrc"
    src.mkdir()
    (src / "k.cu").write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()
    (prof / "p.txt").write_text("header line\n  indented: 7\ntraffic_bytes_per_launch: 1000   (note)\n"
                                f"instructions_per_launch: 2000\nsource_sha256: {sha}\n")
    f = bench.profiled_fields("p.txt", ["k.cu"], profiles_dir=str(prof), csrc_dir=str(src))
    assert f["traffic_bytes_per_launch"] == "1000" and f["instructions_per_launch"] == "2000"
    assert "indented" not in f                                   # indented lines are readings, not fields
    (src / "k.cu").write_text("kernel v2\n")
    assert bench.profiled_fields("p.txt", ["k.cu"], profiles_dir=str(prof), csrc_dir=str(src)) is None
    assert bench.profiled_fields("missing.txt", ["k.cu"], profiles_dir=str(prof), csrc_dir=str(src)) is None


def test_issue_ceiling_arithmetic():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.issue_ceiling(1.0e6, 1.0e-3, sms=2, sm_mhz=1000.0)
    assert r["peak_inst_per_s"] == 2 * 4 * 1e9
    assert r["achieved_inst_per_s"] == 1e9
    assert abs(r["frac"] - 0.125) < 1e-15
    assert abs(r["min_launch_us"] - 125.0) < 1e-9
