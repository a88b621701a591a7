"""bench.py's clock sampler on the CPU, against a fake nvidia-smi that prints timestamped samples.

The sampler must keep the samples around the timed region only, report the
throttle reasons seen there, and still return a sample when the timed region
is shorter than the sampling period.
"""
import datetime
import importlib.util
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


FAKE = r'''#!{py}
import datetime, sys, time
# every 50 ms one sample; clock 1965 MHz except while /tmp flag file says otherwise
t_end = time.time() + 20
while time.time() < t_end:
    now = datetime.datetime.now()
    try:
        state = open("{flag}").read().strip()
    except OSError:
        state = "idle"
    clk, cap = (1965, "Not Active") if state == "busy" else (345, "Not Active")
    if state == "capped":
        clk, cap = 1300, "Active"
    print(f"{{now:%Y/%m/%d %H:%M:%S.%f}}"[:-3] + f", 0, {{clk}}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {{cap}}",
          flush=True)
    time.sleep(0.05)
'''


def _fake_smi(tmp_path, monkeypatch):
    flag = tmp_path / "state"
    flag.write_text("idle")
    d = tmp_path / "bin"
    d.mkdir()
    exe = d / "nvidia-smi"
    exe.write_text(FAKE.format(py=sys.executable, flag=flag))
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{d}{os.pathsep}{os.environ['PATH']}")
    return flag


def test_sampler_keeps_only_the_timed_window(tmp_path, monkeypatch):
    flag = _fake_smi(tmp_path, monkeypatch)
    bench = _bench()
    bench.ClockSampler.PERIOD_S = 0.05
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.6)  # idle samples before the region
    flag.write_text("busy")
    time.sleep(0.1)
    t0 = time.time()
    time.sleep(0.5)
    t1 = time.time()
    s.mark(t0, t1)
    time.sleep(0.1)
    flag.write_text("idle")
    time.sleep(0.5)  # idle samples after the region
    c = s.stop()
    assert c["sm_mhz"] == 1965
    assert c["sm_max_mhz"] == 1965
    assert c["reasons"] == []
    assert c["samples"] >= 5


def test_sampler_short_region_still_has_a_sample_and_sees_power_cap(tmp_path, monkeypatch):
    flag = _fake_smi(tmp_path, monkeypatch)
    flag.write_text("capped")
    bench = _bench()
    bench.ClockSampler.PERIOD_S = 0.05
    s = bench.ClockSampler(0)
    s.start()
    t0 = time.time()
    t1 = t0 + 0.001  # far shorter than the period
    s.mark(t0, t1)
    c = s.stop()
    assert c["samples"] >= 1
    assert c["sm_mhz"] == 1300
    assert c["reasons"] == ["sw_power_cap"]


def test_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    bench = _bench()
    s = bench.ClockSampler(0)
    s.start()
    s.mark(time.time(), time.time())
    c = s.stop()
    assert c["sm_mhz"] is None and c["reasons"] == ["nvidia-smi unavailable"]
