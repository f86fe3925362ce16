"""Host-side logic of bench.py (no GPU): the roofline peak rule, the
committed DRAM-traffic record and its invalidation when a kernel's sources
change, the work split of the CPU-oracle baseline, and the oracle sample of
the small per-tensor workload."""
import hashlib
import json
import os

import pytest

import bench

PK = (6543.1, 1636.3, 1375.0, "measured")   # (HBM GB/s, bf16 burst, bf16 sustained, source)


def test_peak_burst_when_the_clock_holds():
    p, src = bench.choose_peak("tensor", "fp8", {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, PK)
    assert p == pytest.approx(2 * 1636.3) and "burst" in src


def test_peak_sustained_only_when_the_power_cap_pulls_the_clock_down():
    capped = {"sm_mhz": 1635.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    p, src = bench.choose_peak("tensor", "fp8", capped, PK)
    assert p == pytest.approx(2 * 1375.0) and "sustained" in src
    # the cap touched, but the median clock stayed above 90 % of max: burst
    near_max = {"sm_mhz": 1920.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.choose_peak("tensor", "fp8", near_max, PK)[0] == pytest.approx(2 * 1636.3)
    # clocks pulled down without the power cap (a reason-less drop): burst
    assert bench.choose_peak("tensor", "fp8", {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": []},
                             PK)[0] == pytest.approx(2 * 1636.3)


def test_peak_bf16_kernels_and_memory_bound_kernels():
    capped = {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.choose_peak("tensor", "bf16", capped, PK)[0] == pytest.approx(1375.0)
    p, src = bench.choose_peak("hbm", "fp8", capped, PK)
    assert p == pytest.approx(6543.1) and "HBM" in src
    # no sustained figure measured: the burst one stands even under the cap
    assert bench.choose_peak("tensor", "fp8", capped, (6543.1, 1636.3, None, "measured"))[0] == \
        pytest.approx(2 * 1636.3)


def test_recorded_traffic_is_dropped_when_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    rec = {"kv": {"kernel": "k", "dram_bytes_per_launch": 123.0, "sources": ["k.cu"],
                  "sources_sha256": hashlib.sha256(b"kernel v1").hexdigest()}}
    (tmp_path / "profiles" / "roofline_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("kv") == 123.0
    assert bench.recorded_traffic("paged") is None
    src.write_text("kernel v2")
    assert bench.recorded_traffic("kv") is None


def test_committed_traffic_record_matches_the_sources():
    """Every workload in the committed record names sources that exist, so a
    bench line reports either that figure or null -- never a stale one."""
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "roofline_traffic.json")))
    for w, r in rec.items():
        for f in r["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, f)), (w, f)
        assert r["dram_bytes_per_launch"] > 0


def test_chunks_partition_the_range():
    for n in (1, 7, 64, 1000):
        for parts in (1, 3, 16, 5000):
            ch = bench._chunks(n, parts)
            assert ch[0][0] == 0 and ch[-1][1] == n
            assert all(a < b for a, b in ch) and all(ch[i][1] == ch[i + 1][0] for i in range(len(ch) - 1))


def test_every_workload_has_a_config():
    for w in bench.DEFAULT_STEPS:
        assert bench.config_of(w)["workload"]


@pytest.mark.parametrize("workload", list(bench.DEFAULT_STEPS))
def test_cpu_sample_of_every_workload(workload):
    """The oracle sample behind the reference arm and the GPU line's
    cpu_baseline runs for every workload (one thread: a few seconds each)."""
    v, desc = bench.cpu_sample(workload)
    assert v > 0 and desc
