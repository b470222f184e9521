"""Host logic of bench.py: workload selection, byte accounting, the clock
record, whole-job rates, and the stored ncu traffic (no GPU needed)."""
import json
import os

import pytest
import torch

import bench
import workloads


def test_every_named_workload_is_selectable():
    for name in workloads.ALL:
        w = bench.pick_workload(name)
        assert w.name == name
    w = bench.pick_workload("sweep-m512-d64")
    assert (w.m, w.d) == (512, 64)
    assert bench.pick_workload("gqa", 2).B == 2
    # the context-split run times the long workload, its context over the ranks
    assert bench.pick_workload("long-cp") == workloads.ALL["long"]


def test_byte_accounting_matches_the_stated_per_key_sizes():
    w = workloads.ALL["gqa"]
    n = w.B * w.Hkv * w.T
    # 256 B of bf16 key read, 32 B of code + 2 B of norm written per key
    assert bench.quantize_bytes(w, n) == n * 290
    # code + norm + bf16 value row per KV key
    assert bench.decode_bytes(w) == n * 290
    assert bench.decode_bytes(w) == 608174080


def test_whole_job_rate_counts_every_rank():
    # weak scaling: each rank's units over the slowest rank's time
    assert bench.whole_job_rate(1000, 4, 2.0) == pytest.approx(2e6)
    assert bench.reduce_max_over_ranks(3.5, 1, "cpu") == 3.5


def test_clock_record_parsing():
    s = bench.ClockSampler(0)
    for i, line in enumerate([
            "0, 1965, 1965, 240.1, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1950, 1965, 250.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1965, 1965, 245.0, 0x0, Not Active, Not Active, Not Active, Not Active",
            "garbage line"]):
        s.feed(line, t=float(i))
    r = s.summary()
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] == 3
    assert r["power_w_max"] == 250.0
    s = bench.ClockSampler(0)
    s.feed("0, 1200, 1965, 500, 0x8, Active, Not Active, Active, Not Active", t=0.0)
    assert s.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler(0).summary()["reasons"] == ["unavailable"]


def test_clock_samples_are_taken_from_the_region_and_its_continuation():
    # idle samples before the region are left out; samples after it count
    # only up to the end of the top-up that kept the same load
    s = bench.ClockSampler(0)
    line = "0, {mhz}, 1965, 300, 0x0, Not Active, Not Active, Not Active, Not Active"
    s.feed(line.format(mhz=345), t=0.5)               # idle, before the region
    s.t0, s.t1, s.t_end = 1.0, 1.05, 1.4
    s.feed(line.format(mhz=1965), t=1.02)             # inside
    s.feed(line.format(mhz=1950), t=1.2)              # same load, after
    s.feed(line.format(mhz=1965), t=1.3)
    s.feed(line.format(mhz=400), t=2.0)               # after the top-up ended
    r = s.summary()
    assert r["samples_in_region"] == 1 and r["samples_same_load_after"] == 2
    assert r["samples"] == 3 and r["sm_mhz"] == 1965


def test_stored_traffic_is_keyed_to_the_kernel_sources():
    p = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(p) as f:
        d = json.load(f)
    assert d
    for key, e in d.items():
        assert e["dram_bytes_per_launch"] > 0 and e["how"], key
        got = bench.ncu_traffic(key)
        # an entry is served only while its sources are unchanged
        fresh = e["source_hash"] == bench.kernel_source_hash(e["sources"])
        assert (got is not None) == fresh, key
    assert bench.ncu_traffic("no-such-kernel") is None


def test_peaks_are_read_or_fall_back():
    gbs, kind = bench.load_peaks()
    assert gbs > 1000 and kind in ("measured", "fallback")
    tf, tkind = bench.load_tensor_peak()
    assert tf > 100 and tkind


def test_quantizer_roofline_bound_follows_the_ridge():
    # 2 m d flops over (2 d + m/8 + 2) bytes per key: m = 512, d = 64 sits above
    # the ridge of the measured peaks (tensor-bound), the headline shape below
    peak = 6457.7
    t_burst, _, _ = bench.load_tensor_peaks()
    for (m, d), bound in (((512, 64), "tensor"), ((256, 128), "hbm"), ((64, 64), "hbm")):
        w = workloads.SWEEP_BASE.with_(m=m, d=d)
        n = w.n_keys
        qb = bench.quantize_bytes(w, n)
        ms = 1.0
        rec = {"ms": ms, "algorithmic_bytes": qb, "GB_per_s": qb / 1e-3 / 1e9}
        r = bench.roofline_of("quantize", rec, w, peak, "measured", full_size=False, n_keys=n)
        ridge = t_burst * 1e12 / (peak * 1e9)
        assert (2 * m * d / (2 * d + m // 8 + 2) > ridge) == (bound == "tensor")
        assert r["bound"] == bound, (m, d)
        assert r["traffic"] is None               # scaled-down workloads carry none
        if bound == "tensor":
            assert r["unit"] == "TFLOP/s"
            assert r["achieved"] == pytest.approx(2 * m * d * n / 1e-3 / 1e12)
            assert r["frac"] == pytest.approx(r["achieved"] / t_burst)
        else:
            assert r["unit"] == "GB/s" and r["frac"] == pytest.approx(rec["GB_per_s"] / peak)


def test_search_launch_count_follows_the_call_plan():
    # projection + full pass + merge, plus the sample pass and its merge when
    # the index has at least 8 tiles of 256 vectors per CTA; per 128 queries
    assert bench.search_launches_per_call(8388608, 128) == 5
    assert bench.search_launches_per_call(1000, 128) == 3
    assert bench.search_launches_per_call(8388608, 129) == 10
    assert bench.search_launches_per_call(148 * 256 * 8, 1, sms=148) == 5
    assert bench.search_launches_per_call(148 * 256 * 8 - 256, 1, sms=148) == 3
