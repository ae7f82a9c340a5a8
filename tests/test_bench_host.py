"""Host-side rules of bench.py (no GPU needed)."""
import bench


def test_clock_record_rejection():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert not bench.clock_rejected(ok)
    # a power cap is kept; hardware and thermal slowdowns are not
    assert not bench.clock_rejected({"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clock_rejected({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [r]})
    # far below the maximum with no reason: a clock left locked
    assert bench.clock_rejected({"sm_mhz": 1100.0, "sm_max_mhz": 1965.0, "reasons": []})
    # no samples: nothing to reject on
    assert not bench.clock_rejected({"sm_mhz": None, "sm_max_mhz": None,
                                     "reasons": ["clock sampling unavailable"]})


def test_traffic_is_reported_only_for_the_captured_sources_and_shape():
    for kind in ("prefill", "decode"):
        t = bench.TRAFFIC[kind]
        same = t["source_hash"] == bench.source_hash(kind)
        assert bench.traffic(kind, None, t["shape"]) == (t["bytes"] if same else None)
        other = tuple(x + 1 for x in t["shape"])
        assert bench.traffic(kind, None, other) is None
    assert bench.traffic("prefill", 123, (1, 1, 1)) == 123  # an explicit capture overrides
