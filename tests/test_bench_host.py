"""Host-side logic of bench.py that needs no GPU: the timed region replays exactly --steps steps, and the
clock record is taken from the samples inside the timed region."""
import bench


def test_timed_region_replays_exactly_the_requested_steps():
    for n in (1, 5, 20, 63, 64, 65, 128, 130, 19200):
        full, rest = bench.graph_counts(n)
        assert full * bench.GRAPH_STEPS + rest == n and 0 <= rest < bench.GRAPH_STEPS
    assert bench.graph_counts(20) == (0, 20)  # fewer steps than one graph: one graph of exactly 20 steps


def test_clock_record_uses_the_timed_window():
    c = bench.ClockSampler(None)
    c.max_mhz = 1965.0
    # (time, sm MHz, clock-event reasons, watts): a soak at 1500 MHz with the power cap, then the timed region
    c.samples = [(0.0, 1500.0, 0x4, 900.0), (1.0, 1500.0, 0x4, 950.0), (2.0, 1965.0, 0x0, 700.0),
                 (2.5, 1950.0, 0x0, 710.0), (4.0, 1200.0, 0x40, 990.0)]
    c.marks = [1.9, 3.0]
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] in (1950.0, 1965.0) and s["reasons"] == []
    assert s["source"].endswith("timed region")
    c.marks = [5.0, 6.0]  # no sample inside: the whole run is reported, and says so
    s = c.summary()
    assert s["samples"] == 5 and "hw_thermal_slowdown" in s["reasons"] and "sw_power_cap" in s["reasons"]
    assert s["source"].endswith("whole run")
    empty = bench.ClockSampler(None)
    assert empty.summary()["samples"] == 0
