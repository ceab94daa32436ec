"""bench.py's host-side bookkeeping, without a GPU: the ncu traffic lookup (averaged over
a workload's stages, withheld once the GEMM sources differ from the profiled ones), the
algorithmic byte count of select+gather, the kernels launched per step and the summary
of the clock samples (the median SM clock and the throttle reasons seen)."""
import json

import pytest

import bench
from workloads import WORKLOADS


def test_traffic_is_averaged_over_stages_and_withheld_on_other_sources(monkeypatch, tmp_path):
    d = {"entries": [
        {"kernel": "fc1", "workload": "umt_l", "stage": s, "source_hash": "h0",
         "dram_bytes_per_launch": b} for s, b in enumerate((300.0, 200.0, 100.0))]}
    d["entries"].append({"kernel": "fc2", "workload": "umt_l", "stage": 0, "source_hash": "h0",
                         "dram_bytes_per_launch": 50.0})
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(d))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "h0")
    assert bench.ncu_traffic("fc1", "umt_l", 3) == pytest.approx(200.0)
    assert bench.ncu_traffic("fc2", "umt_l", 1) == pytest.approx(50.0)
    assert bench.ncu_traffic("fc2", "umt_l", 3) is None      # stages 1 and 2 missing
    assert bench.ncu_traffic("fc1", "deit_s", 1) is None     # no entry
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "h1")
    assert bench.ncu_traffic("fc1", "umt_l", 3) is None      # taken on other kernels


def test_committed_traffic_entries_cover_every_workload_stage():
    """profiles/traffic.json has one fc1 and one fc2 entry per stage of every workload
    the bench can time (besides the tiny one), all taken on one source hash."""
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    hashes = {e["source_hash"] for e in entries}
    assert len(hashes) == 1
    for name in ("umt_l", "deit_s", "deit_b", "umt_b"):
        stages = WORKLOADS[name].stages
        for kern in ("fc1", "fc2"):
            got = sorted(e["stage"] for e in entries if e["workload"] == name and e["kernel"] == kern)
            assert got == list(range(stages)), (name, kern, got)


def test_select_gather_bytes_by_hand():
    """UMT-L stage 0 (B = 16, L = 1569, C = 1024, keep 1097): 8 partials per row (4 column
    tiles of fc2, 2 groups each), the scores, kept_idx written and read, the kept rows
    read and written."""
    import free_vit_token_b200.rs as rs  # host-only calls: the library loads without a GPU
    assert (rs.rs_num_partials(1024), rs.rs_num_partials(768), rs.rs_num_partials(384)) == (8, 6, 4)
    wl = WORKLOADS["umt_l"]
    M, k = 16 * 1569, 1097
    want = M * 8 * 4 + M * 4 + 16 * (k + 1) * 4 + 16 * (k + 1) * (4 + 2 * 1024 * 2)
    assert bench.select_gather_stage_bytes(rs, wl, 0) == want
    total = sum(bench.select_gather_stage_bytes(rs, wl, s) for s in range(3))
    assert bench.select_gather_bytes(rs, wl) == total


def test_kernels_per_step():
    assert bench.kernels_per_step(WORKLOADS["umt_l"]) == 12
    assert bench.kernels_per_step(WORKLOADS["deit_s"]) == 4


def test_clock_summary_median_and_reasons():
    cs = bench.ClockSampler(0)
    cs._lines = [(1.0, "1965, 1965, 700.0, Not Active, Not Active, Not Active, Not Active"),
                 (2.0, "1700, 1965, 1000.0, Not Active, Not Active, Not Active, Active"),
                 (3.0, "1650, 1965, 1000.0, Not Active, Not Active, Not Active, Active"),
                 (4.0, "garbage line"),
                 (9.0, "900, 1965, 1000.0, Active, Not Active, Not Active, Active")]
    cs.mark_start, cs.mark_end = 1.5, 3.5  # the timed region: the second and third samples
    s = cs.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == pytest.approx(1675.0)
    assert s["sm_max_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]
    cs.mark_start, cs.mark_end = None, None  # all samples: the hardware slowdown shows
    s = cs.summary()
    assert s["samples"] == 4 and "hw_slowdown" in s["reasons"]
