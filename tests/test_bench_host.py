"""Host-side pieces of bench.py that need no GPU: the copy-on-write event of the shared-prompt
workloads and the per-step percentiles."""
import pytest

import bench
import workloads


@pytest.mark.parametrize("name,prompts,samples", [("shared_prefix_4x8", 4, 8),
                                                   ("shared_prefix_16x8", 16, 8),
                                                   ("shared_prefix_16x8_interleaved", 16, 8)])
def test_cow_event_copies_each_prompts_last_shared_block_for_all_sharers_but_one(name, prompts, samples):
    case = workloads.make_case(name, 0)
    pairs = bench.cow_pairs(case).tolist()
    assert len(pairs) == prompts * (samples - 1)
    pb = case.meta["prompt_blocks"]
    tab = case.block_tables.cpu()
    last_shared = {int(tab[s, pb - 1]) for s in range(case.B)}
    private = {int(tab[s, j]) for s in range(case.B) for j in range(pb, tab.shape[1]) if int(tab[s, j]) >= 0}
    assert len(last_shared) == prompts
    srcs = [p[0] for p in pairs]
    dsts = [p[1] for p in pairs]
    assert set(srcs) == last_shared and all(srcs.count(x) == samples - 1 for x in last_shared)
    assert len(set(dsts)) == len(dsts) and set(dsts) <= private     # distinct private blocks
    assert all(0 <= b < case.num_blocks for b in srcs + dsts)


def test_no_cow_event_without_shared_prompts():
    case = workloads.make_case("llama3_8b_b64", 0, B=4)
    assert "prompt_blocks" not in case.meta


def test_percentiles_nearest_rank():
    xs = [float(i) for i in range(1, 101)]                # 1 .. 100
    assert bench.percentiles_ms(xs) == {"p10": 10.0, "p50": 50.0, "p90": 90.0}
    assert bench.percentiles_ms([3.0]) == {"p10": 3.0, "p50": 3.0, "p90": 3.0}
    assert bench.percentiles_ms([]) is None


def test_nvml_poller_summary_keeps_samples_inside_the_window():
    """The NVML clock poller reports only samples taken inside the timed region, with the
    clock-event reasons that were active in any of them (a fake NVML: no GPU here)."""
    import types
    import bench
    p = bench.NvmlPoller.__new__(bench.NvmlPoller)
    p.ok, p.max_sm = True, 1965
    p.nv = types.SimpleNamespace(nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
                                 nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonSwPowerCap=0x4)
    p.rows = [(0.5, 1200, 0x8, 300.0), (1.0, 1965, 0x0, 250.0), (1.2, 1965, 0x4, 260.0), (2.5, 900, 0x40, 100.0)]
    s = p.summary(0.9, 2.0)
    assert s["samples"] == 2 and s["sm_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert s["power_w_max"] == 260.0 and s["sm_max_mhz"] == 1965
    assert p.summary(3.0, 4.0) is None


def test_ncu_traffic_lookup_by_workload_schedule_and_source_hash(tmp_path, monkeypatch):
    """A committed summary names its workload, partition (decode) or schedule (prefill), its
    traffic per launch and the hash of the kernel sources it was taken on; a stale hash or a
    different schedule finds nothing."""
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    h = bench.kernel_source_hash(bench.PREFILL_SOURCES)
    (tmp_path / "a.md").write_text("workload: w1\nschedule: queue\ntraffic_bytes_per_launch: 123\n"
                                   "kernel_source_sha256_16: %s\n" % h)
    (tmp_path / "b.md").write_text("workload: w1\nschedule: grid\ntraffic_bytes_per_launch: 456\n"
                                   "kernel_source_sha256_16: 0000000000000000\n")
    (tmp_path / "c.md").write_text("workload: w2\npartition: 512\ntraffic_bytes_per_launch: 789\n"
                                   "kernel_source_sha256_16: %s\n" % bench.kernel_source_hash())
    assert bench.ncu_traffic_per_launch("w1", schedule="queue", sources=bench.PREFILL_SOURCES) == 123
    assert bench.ncu_traffic_per_launch("w1", schedule="grid", sources=bench.PREFILL_SOURCES) is None   # stale
    assert bench.ncu_traffic_per_launch("w2", 512) == 789
    assert bench.ncu_traffic_per_launch("w2", 1024) is None
    assert bench.ncu_traffic_per_launch("w1", schedule="queue") is None       # decode sources' hash differs


def test_prefill_row_failure_is_reported_not_raised(monkeypatch):
    def boom(args):
        raise RuntimeError("no GPU here")
    monkeypatch.setattr(bench, "run_prefill", boom)
    row = bench.prefill_side_line(bench.parse_args([]))
    assert row["workload"] == bench.PREFILL_SIDE_WORKLOAD and "no GPU here" in row["error"]
