"""The bench line's clock bookkeeping on the CPU: NVML samples are kept
only inside the timed window when there are any there (the idle moments
around a short region read the boost clock), in-kernel probe readings are
added to the summary, and the burst peak is chosen only when every reading
stayed within 5% of the maximum SM clock."""

import bench


class _FakeSampler:
    """Stands in for bench.ClockSampler after its thread has stopped."""

    def __init__(self, samples):
        self.thread = object()
        self.samples = samples
        self.stop_flag = False

    # ClockSampler.stop joins the thread; nothing to join here
    def stop(self, window=None):
        self.thread = type("T", (), {"join": lambda *a, **k: None})()
        return bench.ClockSampler.stop(self, window)


def _samples():
    # (sm_mhz, max_mhz, reasons, t): idle at boost before and after, capped inside
    return ([(1965, 1965, [], 0.5), (1965, 1965, [], 0.9)] +
            [(1500, 1965, ["sw_power_cap"], 1.0 + 0.01 * i) for i in range(5)] +
            [(1965, 1965, [], 2.0)])


def test_window_keeps_the_timed_region_samples():
    c = bench.clock_summary(_FakeSampler(_samples()), (1.0, 1.1))
    assert c["sm_mhz"] == 1500 and c["samples_in_timed_region"] == 5
    assert c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]


def test_without_samples_in_the_window_all_loaded_samples_count():
    # five capped readings and three at boost: the median over all of them
    c = bench.clock_summary(_FakeSampler(_samples()), (5.0, 6.0))
    assert c["samples_in_timed_region"] == 0 and c["sm_mhz"] == 1500 and c["samples"] == 8


def test_probe_readings_join_the_summary_and_decide_the_peak():
    boost = [(1965, 1965, [], 1.0 + 0.01 * i) for i in range(4)]
    c = bench.clock_summary(_FakeSampler(boost), (1.0, 1.1), probe_mhz_timed_end=1962.4,
                            probe_mhz_trace_end=None)
    assert c["probe_mhz_timed_end"] == 1962 and "probe_mhz_trace_end" not in c
    assert bench.clock_held_max(c)
    c = bench.clock_summary(_FakeSampler(boost), (1.0, 1.1), probe_mhz_timed_end=1500.0)
    assert not bench.clock_held_max(c)  # NVML read boost, the kernel saw the cap
    assert not bench.clock_held_max({})
