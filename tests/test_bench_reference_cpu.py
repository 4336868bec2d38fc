"""bench.py's reference arm (the fp64 oracle timed on the host cores) prints
one JSON line with the contract's keys, without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--ref-step-budget", "0.05"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e",
                "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["extrapolated"] is True and line["measured_sample_s_per_step"] > 0
    assert line["cpu_baseline"]["nproc"] >= 1 and "cpu_model" in line["cpu_baseline"]


def _bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_tensor_peak_follows_the_sampled_clocks():
    b = _bench()
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1637.0, "bf16_tflops_sustained": 1386.0, "source": "measured"}
    assert b.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}) == ("burst", 1637.0)
    assert b.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                                 "reasons": ["sw_power_cap"]}) == ("sustained", 1386.0)
    assert b.tensor_peak(peaks, {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": []}) == ("sustained", 1386.0)
    assert b.tensor_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]})[0] == "sustained"


def test_traffic_is_reported_only_for_the_sources_it_was_captured_on(tmp_path, monkeypatch):
    b = _bench()
    f = tmp_path / "traffic.json"
    monkeypatch.setattr(b, "TRAFFIC_FILE", str(f))
    assert b.load_traffic()[0] == {}
    f.write_text(json.dumps({"source_hash": "0" * 64, "command": "c", "bytes_per_launch": {"w": {"k": 1.0}}}))
    assert b.load_traffic()[0] == {}                       # other sources: stale, nothing reported
    f.write_text(json.dumps({"source_hash": b.library_source_hash(), "command": "c",
                             "bytes_per_launch": {"w": {"k": 1.0}}}))
    assert b.load_traffic()[0] == {"w": {"k": 1.0}}
