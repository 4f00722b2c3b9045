"""Host-side pieces of the benchmark, on the CPU: the clock record's parsing
of nvidia-smi samples (median clock, highest max clock, the throttle reasons
that were active) and the traffic lookup, which reports the captured DRAM
bytes only for the captured workload and only while the pair kernel's
sources are the ones the counters were taken on."""
import bench


def line(sm, mx, hw="Not Active", hwt="Not Active", swt="Not Active", pcap="Not Active"):
    return f"0, {sm}, {mx}, 700.5, 0x0, {hw}, {hwt}, {swt}, {pcap}"


def test_clock_summary_median_max_and_reasons():
    s = bench.ClockSampler(0)._summary([line(1965, 1965), line(1950, 1965, pcap="Active"),
                                         line(1965, 1965), "garbage", line("[N/A]", 1965)])
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    s = bench.ClockSampler(0)._summary([line(1200, 1965, hwt="Active", swt="Active")])
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_thermal_slowdown"]
    s = bench.ClockSampler(0)._summary([])
    assert s["sm_mhz"] is None and s["samples"] == 0


def test_clock_window_without_nvidia_smi():
    c = bench.ClockSampler(0)        # never started: no process
    assert c.window(0.0, 1.0)["reasons"] == ["nvidia-smi unavailable"]


def test_traffic_only_for_the_captured_workload_and_sources(monkeypatch):
    import hashlib
    import os
    h = hashlib.sha256()
    for f in ("nl_pairs.cu", "nl_device.cuh"):
        with open(os.path.join(bench.ROOT, "neighbor_list_construction_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    current = dict(bench.PAIR_TRAFFIC, sha256=h.hexdigest())
    monkeypatch.setattr(bench, "PAIR_TRAFFIC", current)
    assert bench.pair_traffic("saltwater10m") == current["bytes"]
    assert bench.pair_traffic("shell10m") is None
    monkeypatch.setattr(bench, "PAIR_TRAFFIC", dict(current, sha256="0" * 64))
    assert bench.pair_traffic("saltwater10m") is None
