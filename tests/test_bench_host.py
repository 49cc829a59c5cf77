"""Host logic of bench.py on the CPU: the kernel-code hash that keeps a DRAM
traffic capture attached to the code it measured, and the reference arm's
JSON line (the CPU oracle on a bounded sample)."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "chunk_causal_attention_block_b200", "csrc")


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _reader(edit=None):
    def read(name):
        with open(os.path.join(CSRC, name)) as f:
            text = f.read()
        return edit(name, text) if edit else text
    return read


def test_kernel_hash_ignores_comments_and_blank_lines_but_not_code():
    bench = _bench()
    base = bench.kernel_source_sha()
    assert bench.kernel_source_sha(_reader()) == base
    commented = _reader(lambda n, t: t.replace("\n", "\n\n// a note\n", 3) if n == "attn_sm100.cu" else t)
    assert bench.kernel_source_sha(commented) == base
    changed = _reader(lambda n, t: t.replace("kStages = kRopeQ ? 3 : 4", "kStages = kRopeQ ? 3 : 5")
                      if n == "attn_sm100.cu" else t)
    assert bench.kernel_source_sha(changed) != base


def test_traffic_capture_is_attached_only_to_the_code_it_measured(monkeypatch):
    bench = _bench()
    got = bench.dram_traffic("wan13b_round")
    assert got is None or got > 431e6  # at least the algorithmic bytes when attached
    monkeypatch.setattr(bench, "kernel_source_sha", lambda read=None: "0000000000000000")
    assert bench.dram_traffic("wan13b_round") is None


def test_reference_arm_line_has_the_contract_fields():
    bench = _bench()

    class Args:
        config, steps, warmup, gpus = "tiny_f32", 1, 0, 1

    line = bench.run_reference(Args, 0, 1)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert bench.run_reference(Args, 1, 2) is None  # other ranks do no work


def test_clock_summary_keeps_only_the_timed_region_and_decodes_reasons():
    bench = _bench()
    rows = [(0.0, 1965, 1965, 300.0, 0x1),      # idle before the region
            (1.0, 1800, 1965, 900.0, 0x4),      # sw_power_cap
            (1.1, 1700, 1965, 950.0, 0x4),
            (1.2, 1650, 1965, 980.0, 0x4 | 0x40),  # plus hw_thermal_slowdown
            (3.0, 1965, 1965, 250.0, 0x1)]      # idle after it
    got = bench.ClockSampler.summarise(rows, 0.5, 2.0)
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1700 and got["sm_min_mhz"] == 1650 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert bench.ClockSampler.summarise(rows, 5.0, 6.0)["reasons"] == ["no samples"]
    assert bench.ClockSampler.summarise(rows)["samples"] == 5


def test_library_context_arm_reports_unavailable_without_a_gpu():
    import json
    import subprocess
    import sys

    import torch
    if torch.cuda.is_available():
        import pytest
        pytest.skip("a GPU is present: the arm would run the library kernels")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "library"], capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "library" and line["unavailable"] == "no CUDA device"


def test_clock_sampler_polls_nvml_inside_the_window(monkeypatch):
    """The sampler's NVML path against a fake NVML: samples are taken while it
    runs, only those inside the window are kept, reasons are decoded."""
    import sys
    import time
    import types

    calls = {"uuid": None}
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 1
    fake.nvmlInit = lambda: None

    def by_uuid(u):
        calls["uuid"] = u
        return "handle"
    fake.nvmlDeviceGetHandleByUUID = by_uuid
    fake.nvmlDeviceGetHandleByIndex = lambda i: "handle"
    fake.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    fake.nvmlDeviceGetClockInfo = lambda h, c: 1605
    fake.nvmlDeviceGetPowerUsage = lambda h: 985000  # mW
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4  # sw_power_cap
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench = _bench()
    s = bench.ClockSampler(0, uuid="0123-abcd")
    s.start()
    assert s.thread is not None, "NVML path not taken"
    time.sleep(0.02)
    t0 = time.perf_counter()
    time.sleep(0.05)
    t1 = time.perf_counter()
    time.sleep(0.02)
    got = s.stop(t0, t1)
    assert calls["uuid"] == "GPU-0123-abcd"
    assert got["samples"] >= 3 and got["sm_mhz"] == 1605 and got["sm_max_mhz"] == 1965
    assert got["power_w_median"] == 985.0 and got["reasons"] == ["sw_power_cap"]
    assert len(s.rows) > got["samples"]  # samples outside the window were taken and dropped
