"""Host-side logic of bench.py (no GPU): argument defaults, the per-workload summary carried under
'also', the traffic records' staleness check, and the measured peaks file."""
import hashlib
import os

import bench


def test_defaults_time_the_headline_workload():
    args = bench.parse_args([])
    assert args.config is None and args.gpus == 1 and args.impl == "ours"
    assert bench.HEADLINE == 4
    assert args.warmup >= 3
    also = [c for c, _, _ in bench.ALSO]
    assert bench.HEADLINE not in also and len(set(also)) == len(also)
    assert set(also) <= {2, 3, 5, 6, 7, 8}


def test_summary_carries_the_roofline_and_traffic():
    line = {"config": {"workload": "w", "us_per_token": 1.5}, "value": 2.0, "unit": "tokens/s", "steps": 3,
            "warmup": 3, "ms_per_step": 0.5,
            "roofline": {"bound": "hbm", "achieved": 1.0, "peak": 2.0, "unit": "GB/s", "frac": 0.5,
                         "traffic": 123.0, "kernel": "k"},
            "e2e": {"value": 1.0}, "clocks": {"sm_mhz": 1}, "gpu_launches": 3, "device_errors": 0}
    out = bench.summary_of(line)
    assert out["roofline_frac"] == 0.5 and out["roofline_traffic"] == 123.0 and out["us_per_token"] == 1.5
    assert out["e2e_value"] == 1.0 and out["gpu_launches"] == 3
    assert bench.summary_of(None) is None


def test_traffic_record_is_dropped_when_the_kernel_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (prof / "traffic.txt").write_text(f"# comment\nx.source = k.cu\nx.sha256 = {digest}\nx.bytes_per_launch = 42\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("x") == 42.0
    assert bench.traffic_from_profiles("missing") is None
    src.write_text("kernel v2\n")
    assert bench.traffic_from_profiles("x") is None


def test_recorded_traffic_entries_are_complete():
    """Every record in profiles/traffic.txt names an existing source, a sha256 and a byte count."""
    path = os.path.join(bench.ROOT, "profiles", "traffic.txt")
    keys = {}
    for line in open(path):
        if line.startswith("#") or "=" not in line:
            continue
        k, v = line.strip().split("=", 1)
        keys[k.strip()] = v.strip()
    names = {k.rsplit(".", 1)[0] for k in keys}
    assert names
    for n in names:
        assert os.path.exists(os.path.join(bench.ROOT, keys[f"{n}.source"]))
        assert len(keys[f"{n}.sha256"]) == 64
        assert float(keys[f"{n}.bytes_per_launch"]) > 0


def test_measured_peaks_are_read():
    peaks = bench.load_peaks()
    assert peaks["hbm_gbs"] > 1000 and peaks["bf16_tflops"] > 100
