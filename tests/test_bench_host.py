"""Host-side pieces of bench.py (no GPU needed): the clock sampler keeps the
samples taken inside the timed region."""
import importlib.util
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


# Stands in for nvidia-smi: one CSV line every 20 ms, the SM clock counting
# up from 1000 MHz, sw_power_cap active on every third line.
FAKE = (
    "import sys, time\n"
    "i = 0\n"
    "while True:\n"
    "    cap = 'Active' if i % 3 == 0 else 'Not Active'\n"
    "    print(f'{1000 + i}, 1965, 500.0, Not Active, Not Active, Not Active, {cap}', flush=True)\n"
    "    i += 1\n"
    "    time.sleep(0.02)\n"
)


def test_clock_sampler_keeps_the_timed_window():
    bench = _bench()
    with bench.ClockSampler(0, cmd=[sys.executable, "-c", FAKE]) as clk:
        assert clk.samples, "sampling runs before the timed region"
        time.sleep(0.1)
        clk.start()
        time.sleep(0.3)
        clk.stop()
        time.sleep(0.1)
    t0, t1 = clk.window
    inside = [ln for t, ln in clk.samples if t0 <= t <= t1]
    s = clk.summary()
    assert s["window"] == "timed region"
    assert 0 < s["samples"] == len(inside) < len(clk.samples)
    clocks = sorted(float(ln.split(",")[0]) for ln in inside)
    assert clocks[0] <= s["sm_mhz"] <= clocks[-1]
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_samples_in_the_window():
    bench = _bench()
    with bench.ClockSampler(0, cmd=[sys.executable, "-c", FAKE]) as clk:
        time.sleep(0.1)
        clk.start()
        clk.stop()
    s = clk.summary()
    assert s["window"] == "whole sampler run" and s["samples"] == len(clk.samples) > 0


def test_clock_sampler_without_nvidia_smi():
    bench = _bench()
    with bench.ClockSampler(0, cmd=["/nonexistent/nvidia-smi"]) as clk:
        clk.start()
        clk.stop()
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"],
                             "samples": 0}
