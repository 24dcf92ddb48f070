"""The algorithmic bytes behind the bench's achieved GB/s (the roofline numerator), derived by
hand per call: packed sign bits N*K/8, the 4-byte tensor scale alpha, x bf16 (2 bytes, read once
per call), y fp32 (4 bytes per row)."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_bitnet_layer_fused_bytes(N, K):
    assert bench.layer_bytes("bitnet", N, K)["fused"] == N * K // 8 + 4 + 2 * K + 4 * N


def test_grouped_calls_read_x_once():
    # q, k, v: three 4096x4096 weight sets, three alphas, three y, one x
    assert bench.call_bytes([4096] * 3, 4096) == 3 * (4096 * 4096 // 8 + 4 + 4 * 4096) + 2 * 4096
    assert bench.call_bytes([4096], 4096) == bench.layer_bytes("bitnet", 4096, 4096)["fused"]


def test_decode_step_bytes_match_the_traffic_record():
    """Per call type, the numerator equals the algorithmic bytes stored beside the DRAM counters,
    and the 32-layer step totals about 816 MB (far above the 126 MB L2)."""
    shapes = {n: (N, K) for n, N, K in bench.LLAMA7B}
    per_call = {}
    for names in bench.LLAMA7B_CALLS:
        K = shapes[names[0]][1]
        assert all(shapes[n][1] == K for n in names)          # a group shares its input
        per_call[names] = bench.call_bytes([shapes[n][0] for n in names], K)
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))["bitnet_fused_llama7b_grouped"]
    stored = rec["per_call_algorithmic_bytes"]
    assert sorted(stored.values()) == sorted(per_call.values())
    step = 32 * sum(per_call.values())
    assert 815e6 < step < 817e6
    # the record's per-launch DRAM figure is the mean over the four call types
    assert rec["dram_bytes_per_launch"] == sum(rec["per_call_dram_bytes"].values()) / 4


def test_clock_parse_reads_median_max_and_reasons():
    """Canned nvidia-smi lines (csv, noheader, nounits): median SM clock, the max clock, and
    each throttle reason that was Active in any sample; malformed or N/A lines are skipped."""
    out = "\n".join([
        "2026/12/02 10:00:00.000, 1965, 1965, 640.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:00.020, 1890, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.040, 1950, 1965, 870.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:00.060, [N/A], 1965, 870.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ])
    c = bench.ClockSampler.parse(out)
    assert (c["sm_mhz"], c["sm_max_mhz"], c["samples"]) == (1950.0, 1965.0, 3)
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 990.1
    hot = out.replace("Not Active, Not Active, Not Active, Active", "Active, Not Active, Active, Not Active")
    assert bench.ClockSampler.parse(hot)["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler.parse("")["samples"] == 0


def test_traffic_record_is_dropped_when_the_kernel_source_changes(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))["bitnet_fused_llama7b_grouped"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["source_hash"])
    assert bench.profile_traffic("bitnet_fused_llama7b_grouped") == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profile_traffic("bitnet_fused_llama7b_grouped") is None
    assert bench.profile_traffic("no_such_kernel") is None


def test_clock_record_prefers_the_timed_window():
    """The bench line's clocks come from the samples inside the timed regions when there are
    any, else from the whole sampled run; reasons seen in any window are kept."""
    timed = {"sm_mhz": 1890.0, "samples": 4, "reasons": ["sw_power_cap"]}
    soak = {"sm_mhz": 1965.0, "samples": 9, "reasons": []}
    whole = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "samples": 14, "reasons": ["sw_power_cap"], "power_w_max": 900.0}
    r = bench.clock_record(dict(whole, timed=timed, soak=soak))
    assert (r["sm_mhz"], r["window"], r["timed_samples"], r["soak_samples"]) == (1890.0, "timed regions", 4, 9)
    assert r["reasons"] == ["sw_power_cap"] and r["sm_max_mhz"] == 1965.0
    r = bench.clock_record(dict(whole, timed={"samples": 0}, soak=soak))
    assert (r["sm_mhz"], r["window"]) == (1950.0, "soak + timed")


def test_clock_stats_take_only_the_window():
    """A config line's clocks are the samples that arrived during its timed replays (plus one
    period after), parsed like the bench line's."""
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    row = "2026/01/01 00:00:00.000, {mhz}, 1965, {w}, 0x0, Not Active, Not Active, Not Active, {cap}\n"
    c.lines = [(10.0, row.format(mhz=1965, w=300, cap="Not Active")),
               (20.1, row.format(mhz=1800, w=990, cap="Active")),
               (20.2, row.format(mhz=1820, w=995, cap="Active")),
               (20.5, row.format(mhz=1900, w=700, cap="Not Active")),
               (30.0, row.format(mhz=1965, w=300, cap="Not Active"))]
    s = c.stats(20.0, 20.4)
    assert s["samples"] == 3 and s["sm_mhz"] == 1820.0 and s["reasons"] == ["sw_power_cap"]
    assert s["power_w_max"] == 995.0
    assert c.stats(40.0, 41.0)["samples"] == 0
