"""Multi-process plumbing of the N-GPU runs, on CPU with gloo (world size 2).

The path shards into independent replicas with no data-path collective; what
runs across ranks is the barrier around a timed region, the max-reduction of
the per-rank time and the whole-job rate computed from it. These tests run
those on two gloo ranks, check that a rank waiting on a peer that never
arrives fails within the group's timeout instead of hanging, and that the
reference arm under torchrun runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from hybrid_local_global_b200 import dist as hdist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))


def _worker_max(rank, world, port, out_dir):
    _env(rank, world, port)
    r = hdist.setup("gloo", timeout_s=60)
    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    r.barrier()
    m = r.max_over_ranks(ms)
    rate = hdist.whole_job_rate(units_per_rank=100.0, steps=4, max_ms=m, world=r.world)
    with open(os.path.join(out_dir, "r%d.json" % rank), "w") as f:
        json.dump({"max": m, "rate": rate, "world": r.world, "rank": r.rank}, f)
    r.close()


def test_max_over_ranks_and_rate_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_worker_max, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn")
    got = [json.load(open(tmp_path / ("r%d.json" % r))) for r in range(2)]
    for g in got:
        assert g["world"] == 2
        assert g["max"] == 15.0                       # the slowest rank's time, on every rank
        assert g["rate"] == pytest.approx(2 * 100.0 * 4 / 0.015)


def _worker_dead_peer(rank, world, port, out_dir):
    _env(rank, world, port)
    r = hdist.setup("gloo", timeout_s=3)
    if rank == 1:
        r.close()  # leaves between steps, before the next collective
        return
    err = ""
    try:
        r.barrier()
    except Exception as e:  # the group's timeout ends the wait with an error
        err = type(e).__name__
    with open(os.path.join(out_dir, "dead.json"), "w") as f:
        json.dump({"error": err}, f)


def test_barrier_with_dead_peer_fails_instead_of_hanging(tmp_path):
    port = _free_port()
    ctx = mp.start_processes(_worker_dead_peer, args=(2, port, str(tmp_path)), nprocs=2,
                             start_method="spawn", join=False)
    for p in ctx.processes:
        p.join(timeout=120)
        assert not p.is_alive(), "a rank is still waiting"
    got = json.load(open(tmp_path / "dead.json"))
    assert got["error"], "rank 0's barrier returned although its peer never arrived"


def test_single_process_needs_no_group():
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    r = hdist.setup("gloo")
    assert (r.world, r.rank) == (1, 0)
    assert r.max_over_ranks(3.5) == 3.5
    r.barrier()
    r.close()
    with pytest.raises(ValueError):
        hdist.whole_job_rate(1.0, 1, 0.0, 1)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--ref-rows-local", "2", "--ref-rows-global", "2",
           "--workload", "local_s1024"]
    p = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    if rank == 0:
        assert len(lines) == 1
        line = json.loads(lines[0])
        assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
