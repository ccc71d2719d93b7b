"""Host-side logic of bench.py, on the CPU: the algorithmic FLOP counts of
the Phase-1 roofline, the DRAM-traffic records and their source-hash guard,
the clock summary taken during the timed region, and the whole-job rate."""
import hashlib
import os

import numpy as np
import pytest

import bench
import oracle
from long_context_blockwise_max_b200 import workloads


@pytest.mark.parametrize("wname,pulsar_tf,star_tf", [
    ("LLAMA_32K", 3.18, 7.15),
    ("LLAMA_128K", 37.98, 63.77),
])
def test_attn_flops_match_the_layout_and_the_stated_totals(wname, pulsar_tf, star_tf):
    # bench.py counts 4 d Hq n (n + 1) / 2 per host from closed-form host
    # lengths; the oracle builds each host's rows position by position.  Both
    # must agree, and the totals are the figures the workloads are quoted with.
    w = getattr(workloads, wname)
    sel = np.tile(np.arange(w.k_chunks, dtype=np.int64), (w.n_blocks, 1))
    for star, stated in ((False, pulsar_tf), (True, star_tf)):
        pos = oracle.host_positions(w.L, w.block, 0 if star else w.sink, w.chunk,
                                    np.zeros((w.n_blocks, 0), dtype=np.int64) if star else sel, star=star)
        lengths = [len(p) for p in pos]
        assert lengths == bench.host_lengths(w, star)
        flops = sum(4.0 * w.d * w.hq * n * (n + 1) / 2.0 for n in lengths)
        assert flops == bench.attn_flops(w, star)
        assert abs(flops / 1e12 - stated) < 0.006


def _write_record(path, kernel, workload, sources, sha, rd, wr):
    path.write_text(f"# test record\nkernel {kernel}\nworkload {workload}\nsources {sources}\n"
                    f"sources_sha256 {sha}\ndram_bytes_read {rd}\ndram_bytes_write {wr}\n")


def test_recorded_traffic_is_dropped_once_the_sources_change(tmp_path, monkeypatch):
    src = "include/pulsar.h"
    sha = hashlib.sha256(open(os.path.join(bench.ROOT, src), "rb").read()).hexdigest()
    rec = tmp_path / "traffic.txt"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    _write_record(rec, "k1", "w1", src, sha, 100, 23)
    assert bench.recorded_traffic("k1", "w1") == 123
    assert bench.recorded_traffic("k1", "other") is None
    assert bench.recorded_traffic("k2", "w1") is None
    _write_record(rec, "k1", "w1", src, "0" * 64, 100, 23)   # taken on other sources
    assert bench.recorded_traffic("k1", "w1") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert bench.recorded_traffic("k1", "w1") is None


def test_committed_traffic_records_parse():
    # every record in profiles/roofline_traffic.txt names existing sources and
    # whole byte counts (whether it still matches the sources is checked at
    # bench time)
    records = []
    for line in open(bench.TRAFFIC_FILE):
        line = line.strip()
        if line and not line.startswith("#"):
            key, _, val = line.partition(" ")
            if key == "kernel":
                records.append({})
            records[-1][key] = val.strip()
    assert {r["kernel"] for r in records} == {"phase1_tc_kernel", "phase2_tc_kernel"}
    for r in records:
        for rel in r["sources"].split():
            assert os.path.exists(os.path.join(bench.ROOT, rel)), rel
        assert len(r["sources_sha256"]) == 64
        assert int(r["dram_bytes_read"]) > 0 and int(r["dram_bytes_write"]) > 0


def test_clock_summary_reads_median_max_and_active_reasons():
    c = bench.ClockSampler(0)
    c.out = "\n".join([
        "2026/12/03 05:41:00.000, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 05:41:00.050, 1800, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 05:41:00.100, 1700, 1965, 1001.2, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 05:41:00.150, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",  # unreadable
        "garbage",
    ])
    # no window marked: every readable sample, flagged as such
    s = c.summary()
    assert s == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3,
                 "in_window": False}
    # a window holding the last two samples only (timestamps are host-local time)
    t1 = bench.ClockSampler._epoch("2026/12/03 05:41:00.040")
    t2 = bench.ClockSampler._epoch("2026/12/03 05:41:00.120")
    c.t_start, c.t_end = t1, t2
    assert c.summary() == {"sm_mhz": 1750.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2,
                           "in_window": True}
    # a window with no sample in it falls back to all of them
    c.t_start, c.t_end = t2 + 10, t2 + 11
    assert c.summary()["samples"] == 3 and c.summary()["in_window"] is False
    c.out = ""
    assert c.summary()["samples"] == 0


def test_whole_job_rate_counts_every_rank():
    assert bench.whole_job_rate(131072, 1, 37.0) == pytest.approx(131072 / 0.037)
    assert bench.whole_job_rate(131072, 8, 40.0) == pytest.approx(8 * 131072 / 0.040)


def test_attn_flops_of_host_ranges_add_up():
    # --layout hosts: each rank's roofline counts the FLOPs of its own hosts;
    # the ranks' ranges tile the sequence, so their FLOPs add up to the whole
    from long_context_blockwise_max_b200.distributed import shard_ranges
    w = workloads.LLAMA_128K
    for world in (1, 2, 3, 8):
        parts = [bench.attn_flops(w, hosts=r) for r in shard_ranges(w.n_blocks, world)]
        assert sum(parts) == pytest.approx(bench.attn_flops(w), rel=1e-12)
    # the last host alone: n = 64 + 7 * 2048 + 16384 rows
    n = 64 + 7 * 2048 + 16384
    assert bench.attn_flops(w, hosts=(7, 8)) == 4.0 * w.d * w.hq * n * (n + 1) / 2.0
