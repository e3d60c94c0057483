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
