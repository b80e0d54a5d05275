"""Host-side measurement logic of bench.py, on CPU: the ncu traffic record is reported only for the
kernel source it was captured from, the clock record is read the way the timing rules ask, and the
roofline names the kernel the library dispatches to."""

import sys

import pytest

from conftest import ROOT


@pytest.fixture
def bench(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    sys.path.insert(0, ROOT)
    import bench as b
    return b


def test_traffic_record_follows_the_kernel_source(bench, monkeypatch):
    rec = dict(ln.split(": ", 1) for ln in open(bench.TRAFFIC_FILE).read().splitlines()
               if ln and not ln.startswith("#"))
    # the captured kernels, per cache format
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kv="bf16": rec[f"kernel_source_sha.{kv}"])
    for kv in ("bf16", "fp8"):
        t, src = bench.recorded_traffic("mixed", kv)
        assert t == (int(rec[f"mixed.{kv}.dram_bytes_read_per_launch"]) +
                     int(rec[f"mixed.{kv}.dram_bytes_write_per_launch"]))
        # the source names the committed record and the command that made it
        assert src.startswith("profiles/decode_kernel_traffic.txt") and "gpurun_out" not in src.split("(")[0]
        assert "ncu" in src and "--clock-control none" in src and "bench.py" in src
        # traffic must be a little above the algorithmic bytes (no re-reads), never below
        alg = int(rec[f"mixed.{kv}.algorithmic_bytes_per_launch"])
        assert alg <= int(rec[f"mixed.{kv}.dram_bytes_read_per_launch"]) <= 1.02 * alg
    assert bench.recorded_traffic("mixed", "bf16", q_len=2)[0] is None  # no capture for multi-query
    assert bench.recorded_traffic("no_such_workload", "bf16")[0] is None
    # a change to one format's kernel voids that format's record only
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda kv="bf16": "0" * 16 if kv == "fp8" else rec["kernel_source_sha.bf16"])
    t, why = bench.recorded_traffic("mixed", "fp8")
    assert t is None and "changed" in why
    assert bench.recorded_traffic("mixed", "bf16")[0] is not None


def test_kernel_source_hash_covers_each_format_sources(bench):
    import hashlib
    import os
    for kv in ("bf16", "fp8"):
        h = hashlib.sha256()
        for rel in bench.KERNEL_SOURCES[kv]:
            h.update(open(os.path.join(bench.ROOT, rel), "rb").read())
        assert bench.kernel_source_hash(kv) == h.hexdigest()[:16]
    assert any("decode_tc.cu" in f for f in bench.KERNEL_SOURCES["fp8"])
    assert not any("decode_tc.cu" in f for f in bench.KERNEL_SOURCES["bf16"])


def test_step_statistics(bench):
    s = bench.step_stats([0.1, 0.2, 0.3, 0.4, 0.5])
    assert s == {"median": 300.0, "p10": 140.0, "p90": 460.0}


def test_clock_record_summary(bench, tmp_path):
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.file = open(tmp_path / "clocks.csv", "w+")
    rows = ["0, 600, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active",  # idle, before load
            "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    cs.file.write("\n".join(rows) + "\n")
    s = cs.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0  # median under load; the idle sample is left out
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4 and s["power_w_max"] == 990.0
    cs.file.seek(0)
    cs.file.truncate()
    cs.file.write("0, 1400, 1965, 900.0, 0x0, Active, Not Active, Not Active, Not Active\n")
    assert cs.summary()["reasons"] == ["hw_slowdown"]  # a run the timing rules reject
    cs.file.seek(0)
    cs.file.truncate()
    assert cs.summary()["samples"] == 0


def test_roofline_names_the_dispatched_kernel(bench):
    from variable_length_paged_b200 import workloads as W
    mixed = W.Problem(batch=32, num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=64, max_pages_per_req=250,
                      num_pages=8400, scale=0.088)
    assert bench.decode_kernel_name(mixed, False, 1) == "decode_kernel<128,bf16>"
    assert bench.decode_kernel_name(mixed, True, 1).startswith("decode_tc_kernel")  # FP8 plain decode: tcgen05
    assert bench.decode_kernel_name(mixed, True, 2) == "decode_kernel<128,fp8>"  # FP8 multi-query: warp MMA
