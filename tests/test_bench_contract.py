"""The benchmark's command-line contract, on the CPU: the reference arm (the oracle
as it stands) prints one JSON line with the keys the contract names, and too few
warm-up steps are refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=600, cwd=ROOT)


def test_reference_arm_prints_the_contract_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--config", "0")
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert "workload" in line["config"]


def test_too_few_warmup_steps_are_refused():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "2", "--config", "0")
    assert r.returncode != 0


def test_traffic_record_from_ncu_raw_csv(tmp_path, monkeypatch):
    """--record-traffic reads ncu's raw CSV page (a header row of metric names, a
    row of units, one row per launch) and writes the mean DRAM bytes per verify
    launch with the kernel source hash; measured_traffic reads it back only while
    the hash matches."""
    sys.path.insert(0, ROOT)
    import bench
    csv_path = tmp_path / "raw.csv"
    csv_path.write_text(
        '"ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum"\n'
        '"","","Mbyte","Gbyte"\n'
        '"0","ddt::build_mask_kernel(const int *)","1.00","0.001"\n'
        '"1","ddt::verify_attn_kernel(CUtensorMap_st, ddt::VerifyParams)","460.00","0.1187"\n'
        '"2","ddt::verify_attn_kernel(CUtensorMap_st, ddt::VerifyParams)","462.00","0.1189"\n')
    rec_path = tmp_path / "rec.json"
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(rec_path))
    assert bench.record_traffic(str(csv_path), "ncu ...") == 0
    rec = json.loads(rec_path.read_text())
    assert rec["launches"] == 2
    assert abs(rec["traffic_bytes_per_launch"] - (461.0e6 + 118.8e6)) < 1.0
    assert bench.measured_traffic(2) == rec["traffic_bytes_per_launch"]
    assert bench.measured_traffic(3) is None
    rec["kernel_source_sha256"] = "0" * 64
    rec_path.write_text(json.dumps(rec))
    assert bench.measured_traffic(2) is None


def test_clock_summary_takes_samples_inside_the_timed_region():
    """The NVML samples inside the marked region decide the clock summary (median
    SM MHz, the union of the throttle reasons); with fewer than three of them the
    nvidia-smi samples do."""
    sys.path.insert(0, ROOT)
    import bench

    c = bench.ClockSampler("0")
    c.nvml_max = 1965.0
    c.region = (10.0, 10.05)
    c.nvml_samples = [(9.99, 1965.0, 0), (10.01, 1500.0, 0x4), (10.02, 1520.0, 0x4),
                      (10.03, 1480.0, 0x4 | 0x40), (10.06, 1965.0, 0)]
    s = c.summary()
    assert s["sm_mhz"] == 1500.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    c.region = (10.0, 10.015)
    c.lines = ["0, 1965, 1965, 300, 0x0, Not Active, Not Active, Not Active, Active"]
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]
    assert s["source"].startswith("nvidia-smi")


def test_sustained_peak_only_for_a_power_capped_region():
    """The burst peak is the roofline's denominator unless the timed region ran
    power-capped: longer than 2 s, or NVML samples inside it with sw_power_cap
    and the median SM clock below 95 % of its maximum."""
    sys.path.insert(0, ROOT)
    import bench

    peaks = {"bf16_tflops": 1631.8, "bf16_tflops_sustained": 1400.0}
    nvml = "NVML every ~2 ms inside the timed region"
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "source": nvml}
    capped = {"sm_mhz": 1567.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "source": nvml}
    assert bench.choose_peak(peaks, 0.05, full)[:2] == (1631.8, False)
    assert bench.choose_peak(peaks, 0.3, capped)[:2] == (1400.0, True)
    assert "power-capped" in bench.choose_peak(peaks, 0.3, capped)[2]
    assert bench.choose_peak(peaks, 3.0, full)[:2] == (1400.0, True)
    # the cap bit alone at full clock, or samples from outside the region, do not switch
    assert bench.choose_peak(peaks, 0.3, dict(capped, sm_mhz=1940.0))[:2] == (1631.8, False)
    smi = dict(capped, source="nvidia-smi every 100 ms around the timed region")
    assert bench.choose_peak(peaks, 0.3, smi)[:2] == (1631.8, False)
