"""The bench's multi-rank plumbing (one process per GPU; replicas, no data-path collective):
rendezvous, barrier, the max over ranks of the device time and the whole-job rate, run as two
gloo ranks on the host."""
import os
import socket
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="host-side ranks (gloo) only")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, _ = bench.dist_setup()
    bench.barrier(w)
    ms = bench.max_over_ranks(w, 10.0 + 5.0 * r)          # rank 1 is the slower one
    q.put((r, w, dist.get_backend(), ms, bench.aggregate_rate(w, 1, ms)))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1]
    for _, world, backend, ms, rate in got:
        assert world == 2 and backend == "gloo"
        assert ms == 15.0                                  # the slower rank's time on both ranks
        assert rate == pytest.approx(2 / 15e-3)            # both ranks' work over that time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1, 3.5) == 3.5
    assert bench.aggregate_rate(1, 4, 2.0) == pytest.approx(2000.0)


def test_reference_arm_under_two_ranks_prints_one_line():
    """`bench.py --impl reference` launched as two ranks: rank 0 times the oracle and prints the
    one JSON line; rank 1 exits without work; both exit 0."""
    import json
    import subprocess
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
