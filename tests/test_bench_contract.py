"""bench.py's configuration list and command line, on CPU: every measured layer
configuration of the workloads is in the configs record, the default run is the
headline decode workload, and the command line parses."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_mixture_experts_top_b200.workloads import WORKLOADS  # noqa: E402


def test_configs_record_covers_every_workload_size():
    want = {(name, T) for name, w in WORKLOADS.items() if name != "tiny_mxfp4" for T in w.tokens}
    assert want == set(bench.CONFIGS)
    assert len(bench.CONFIGS) == len(set(bench.CONFIGS))


def test_default_run_is_the_headline_decode_workload():
    w = WORKLOADS[bench.WORKLOAD]
    assert w.fmt == "nf4" and max(w.tokens) == 64 and not w.lora_rank


def test_command_line_parses():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    for flag in ("--gpus", "--steps", "--warmup", "--impl", "--only-config", "--no-configs"):
        assert flag in r.stdout


def test_clock_sampler_samples_a_short_region(monkeypatch):
    """A 2.4 ms region whose host thread holds the interpreter, then waits (as a timed region of
    20 decode steps does) gets several samples; the interpreter's switch interval is restored."""
    import time
    import types
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 1
    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByIndex = lambda i: object()
    fake.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    fake.nvmlDeviceGetClockInfo = lambda h, c: 1900
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 | 0x1
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    before = sys.getswitchinterval()
    c = bench.ClockSampler(0)
    c.start()
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < 0.0024:
        n += 1
    time.sleep(0.002)
    rec = c.summary()
    assert rec["samples"] >= 3 and rec["sm_mhz"] == 1900 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]          # gpu_idle is not reported
    assert sys.getswitchinterval() == before
