"""Host logic of bench.py, without a GPU: the reference arm's JSON line, the
roofline arithmetic against the measured peaks, the DRAM-traffic lookup
gated on the kernel source's sha256, replica aggregation and the workload
configurations."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run_bench(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       env=e, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout


def test_reference_arm_json_line():
    out = _run_bench(["--impl", "reference", "--workload", "frac35", "--steps", "1", "--warmup", "0"])
    lines = [ln for ln in out.splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference"
    assert j["metric"] == bench.WORKLOAD_METRICS["frac35"]
    assert j["unit"] == "units/s" and j["higher_is_better"] is True
    assert j["value"] > 0 and j["steps"] == 1 and j["warmup"] == 0 and j["n_gpus"] == 1
    assert j["config"]["workload"] == bench.WORKLOAD_NAMES["frac35"]
    assert "model" not in j["config"]
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["cpu_baseline"]["cores"] >= 1 and j["cpu_baseline"]["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "units/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    out = _run_bench(["--impl", "reference", "--workload", "frac35", "--steps", "1", "--warmup", "0"],
                     env={"RANK": "1", "WORLD_SIZE": "2"})
    assert out.strip() == ""


def test_roofline_arithmetic_against_measured_peaks():
    hbm, bf16, bf16s, src = bench._peaks()
    peaks = {"hbm_gbs": hbm, "bf16_tflops": bf16, "bf16_tflops_sustained": bf16s}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):                # the driver's measurement, else the stated fallback
        with open(path) as f:
            j = json.load(f)
        assert src == "measured" and hbm == float(j["hbm_gbs"]) and bf16 == float(j["bf16_tflops"])
    else:
        assert src == "fallback" and hbm == bench.FALLBACK_HBM_GBS
    op = bench.Op("x", None, 1, "u", "hbm", 3_000_000_000, "k", 1)       # bytes moved in one launch
    r = bench.roofline_of(op, 1.0)                                         # ... in 1 ms = 3000 GB/s
    assert r["unit"] == "GB/s" and r["peak"] == peaks["hbm_gbs"]
    assert abs(r["achieved"] - 3000.0) < 0.01 and abs(r["frac"] - 3000.0 / peaks["hbm_gbs"]) < 1e-4
    assert r["algorithmic_bytes"] == 3_000_000_000 and r["traffic"] is None
    op_t = bench.Op("y", None, 1, "u", "tensor", 2e12, "k", 1, peak="sustained")
    r = bench.roofline_of(op_t, 2.0)                                       # 2 TFLOP in 2 ms = 1000 TFLOP/s
    assert r["unit"] == "TFLOP/s" and r["peak"] == peaks["bf16_tflops_sustained"]
    assert abs(r["achieved"] - 1000.0) < 1e-6 and abs(r["frac"] - 1000.0 / peaks["bf16_tflops_sustained"]) < 1e-4
    op_b = bench.Op("z", None, 1, "u", "tensor", 2e12, "k", 1, peak="burst")
    assert bench.roofline_of(op_b, 2.0)["peak"] == peaks["bf16_tflops"]


def test_traffic_lookup_is_gated_on_the_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"// a kernel\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    entries = {"w/op": {"source": "kernel.cu", "sha256": sha, "bytes_per_launch": 12345},
               "w/stale": {"source": "kernel.cu", "sha256": "0" * 64, "bytes_per_launch": 777}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"entries": entries}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("w/op") == 12345
    assert bench.traffic_for("w/stale") is None
    assert bench.traffic_for("w/missing") is None
    assert bench.traffic_for(None) is None
    src.write_bytes(b"// the kernel, changed\n")
    assert bench.traffic_for("w/op") is None


def test_committed_traffic_entries_are_well_formed():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    assert entries
    for key, e in entries.items():
        assert os.path.exists(os.path.join(ROOT, e["source"])), key
        assert os.path.exists(os.path.join(ROOT, e["summary"])), key
        assert len(e["sha256"]) == 64 and e["bytes_per_launch"] > 0, key
        assert "ncu" in e["command"] and "--clock-control none" in e["command"], key
        scaled = (e["dram_read_bytes"] + e["dram_write_bytes"]) * e["workload_units"] / e["captured_units"]
        assert abs(scaled - e["bytes_per_launch"]) <= 1 + 1e-9 * scaled, key


@pytest.mark.parametrize("times", [[1.0], [1.0, 2.0], [0.5, 0.25, 0.75, 0.5]])
def test_replica_aggregate_is_all_units_over_the_slowest_rank(times):
    value, t = bench.aggregate(1000.0, times)
    assert t == max(times)
    assert abs(value - 1000.0 * len(times) / max(times)) < 1e-9


@pytest.mark.parametrize("workload", sorted(bench.WORKLOADS))
def test_workload_configs(workload):
    cfg = bench.workload_config(workload, {})
    assert cfg["workload"] == bench.WORKLOAD_NAMES[workload]
    assert cfg["parallelism"] == "replicas" and "model" not in cfg
    assert workload in bench.WORKLOAD_METRICS and workload in bench.UNIT_NOTES
    assert workload in bench.SAMPLE_TEXT and workload in bench.SAMPLE_L
    json.dumps(cfg)


class _FakeNVML:
    """Read-only NVML stand-in: scripted SM clocks, power and throttle
    reasons; any other attribute (a setter, a reset) is recorded as a
    violation and fails."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20

    def __init__(self, reasons):
        self.calls, self.violations, self.reasons, self.n = [], [], reasons, 0

    def nvmlInit(self):
        self.calls.append("init")

    def nvmlDeviceGetHandleByUUID(self, sel):
        raise RuntimeError("no such uuid")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("handle", i)

    def nvmlDeviceGetClockInfo(self, h, which):
        self.n += 1
        return (1965, 1965, 1800)[self.n % 3]

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetPowerUsage(self, h):
        return 512_000                     # mW

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons

    def __getattr__(self, name):
        self.violations.append(name)
        raise AttributeError(name)


def test_clock_sampler_reads_nvml_and_changes_nothing(monkeypatch):
    import time
    import types
    fake = _FakeNVML(reasons=_FakeNVML.nvmlClocksEventReasonSwPowerCap)
    mod = types.ModuleType("pynvml")
    for k in dir(_FakeNVML):
        if k.startswith("nvml") or k.startswith("NVML"):
            setattr(mod, k, getattr(fake, k))
    mod.__getattr__ = fake.__getattr__
    monkeypatch.setitem(sys.modules, "pynvml", mod)
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.05)
    r = s.stop()
    assert r["source"].startswith("nvml")
    assert r["samples"] >= 5 and r["sm_mhz"] in (1800.0, 1965.0) and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 512.0
    assert fake.violations == []


def test_clock_sampler_parses_nvidia_smi_lines(tmp_path):
    csv_path = tmp_path / "clocks.csv"
    csv_path.write_text("0, 1965, 1965, 700.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                        "0, 1950, 1965, 810.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                        "0, 1800, 1965, 990.1, 0x0000000000000024, Not Active, Not Active, Active, Active\n"
                        "garbage line\n")

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.thread, s.nvml, s.proc, s.path, s.reasons = None, None, _Proc(), str(csv_path), set()
    r = s.stop()
    assert r["source"].startswith("nvidia-smi")
    assert r["samples"] == 3 and r["sm_mhz"] == 1950.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"] and r["power_w_max"] == 990.1
    assert not csv_path.exists()
