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
