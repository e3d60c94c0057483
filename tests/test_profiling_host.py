"""Host-side checks of the profiling helpers: the ncu launch-list fold and
the traffic records bench.py reads from profiles/ (no GPU, no ncu)."""
import os

from hybrid_local_global_b200 import profiling

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_launch_list_fold(tmp_path):
    p = tmp_path / "l.csv"
    p.write_text(
        '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
        '"0","void hlg::(anonymous namespace)::k_a<256>(Args)","gpu__time_duration.sum","nsecond","1,000"\n'
        '"1","void unnamed>::k_b(Args)","gpu__time_duration.sum","usecond","3"\n'
        '"2","void hlg::(anonymous namespace)::k_a<256>(Args)","gpu__time_duration.sum","nsecond","2000"\n')
    out = profiling.summarize_launches(str(p)).splitlines()
    assert out[1].split()[:5] == ["k_a<256>", "2", "3.0", "1.50", "50.00%"]
    assert out[2].split()[:5] == ["k_b", "1", "3.0", "3.00", "50.00%"]


def test_traffic_records_match_current_sources():
    recs = profiling.traffic_records(os.path.join(ROOT, "profiles"))
    assert recs, "profiles/ carries no traffic-record line"
    for r in recs:
        assert r["kernel"] in profiling.KERNEL_SOURCES
        assert int(r["bytes"]) > 0
        assert len(r["digest"]) == 16


def test_parity_summary_of_the_cpu_baselines():
    """bench.py's parity figures: the largest and the mean absolute error over
    every element compared, rows counted by the reference's last dimension,
    judged against the tests' tolerance (max 2e-2, mean 2e-3); a non-finite
    GPU value fails it."""
    import numpy as np
    import bench
    p = bench.Parity()
    ref = np.zeros((3, 4))
    p.add(ref + 0.01, ref)
    p.add(np.full(4, 0.001), np.zeros(4))
    s = p.summary("x")
    assert s["rows"] == 4 and abs(s["max_abs"] - 0.01) < 1e-12
    assert abs(s["mean_abs"] - (12 * 0.01 + 4 * 0.001) / 16) < 1e-9
    assert s["within_tolerance"] is False  # mean 7.8e-3 > 2e-3
    q = bench.Parity()
    q.add(np.full((2, 8), 0.015), np.zeros((2, 8)))
    q.add(np.zeros((30, 8)), np.zeros((30, 8)))
    assert q.summary("x")["within_tolerance"] is True
    r = bench.Parity()
    r.add(np.array([[np.nan, 0.0]]), np.zeros((1, 2)))
    assert r.summary("x")["within_tolerance"] is False


def test_stale_traffic_record_is_named():
    """A capture whose digest no longer matches the built sources is not used,
    and the note says which file holds it."""
    import bench
    from hybrid_local_global_b200.profiling import kernel_digest, traffic_records
    recs = traffic_records(os.path.join(ROOT, "profiles"))
    for kernel in sorted({r["kernel"] for r in recs}):
        stale = [r for r in recs if r["kernel"] == kernel and r.get("digest") != kernel_digest(kernel)]
        note = bench.no_traffic_note(kernel)
        if stale:
            assert all(r["file"] in note for r in stale)
            assert all(r.get("digest") != kernel_digest(kernel) for r in stale)
        else:
            assert note == "no ncu capture of the current kernel sources"


def test_clock_rejection_rule():
    """Hardware and thermal slowdowns disqualify a timed region, and so does
    a clock well below its maximum with no reason; the power cap alone does
    not."""
    import bench
    ok = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    assert not bench.clock_rejected(ok)
    assert not bench.clock_rejected({"sm_mhz": 1635, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    assert not bench.clock_rejected({"sm_mhz": 1200, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clock_rejected({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [r, "sw_power_cap"]})
    assert bench.clock_rejected({"sm_mhz": 1100, "sm_max_mhz": 1965, "reasons": []})
    assert bench.clock_rejected({"sm_mhz": 1100, "sm_max_mhz": 1965, "reasons": ["applications_clocks"]})
    assert not bench.clock_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no samples"})


def test_rejected_clock_record_is_measured_again_once(monkeypatch):
    """timed_passes repeats the measurement once when any rank's clock record
    is disqualified, keeps the second, and records the first; the repeat is
    decided from the value reduced over the ranks."""
    import bench

    class Clk:
        def __init__(self, summ):
            self.summ = summ

        def summary(self):
            out = dict(self.summ)
            if getattr(self, "rejected_first", None) is not None:
                out["rejected_first_attempt"] = self.rejected_first
            return out

    bad = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]}
    good = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    for records, other_rank_bad, want_calls in (([good], 0.0, 1), ([bad, good], 0.0, 2),
                                                ([good, good], 1.0, 2), ([bad, bad], 0.0, 2)):
        calls = []

        def once(*a, **k):
            calls.append(1)
            return (10.0 * len(calls), 1.0, {}, Clk(records[len(calls) - 1]))

        monkeypatch.setattr(bench, "timed_passes_once", once)
        monkeypatch.setattr(bench, "max_over_ranks", lambda x, world: max(x, other_rank_bad))
        ms, _, _, clk = bench.timed_passes(None, None, None, 2, None)
        assert len(calls) == want_calls
        assert ms == 10.0 * want_calls
        if want_calls == 2:
            assert "rejected_first_attempt" in clk.summary()
        else:
            assert "rejected_first_attempt" not in clk.summary()
