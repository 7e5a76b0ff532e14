"""Host logic of bench.py's multi-process (replica) mode, on CPU with gloo.

Every rank runs the same workload independently (no collective in the data
path); the ranks only meet for the barrier around the timed region and for
the max / sum reductions of the timing and the unit counts.  These tests run
that plumbing with two gloo ranks on the host.
"""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    d = bench.Dist(world)
    out = {"world": d.world, "rank": d.rank}
    d.barrier()
    out["max"] = d.max(float(rank + 1))          # timing: the slowest rank decides
    out["sum"] = d.sum(10.0 * (rank + 1))        # units: every rank's work counts
    d.barrier()
    d.close()
    results[rank] = out


def _reference_rank(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    if rank == 0:
        # rank 0 would time the oracle for a minute; here it only joins and leaves
        d = bench.Dist(world)
        d.close()
        results[rank] = ""
        return
    sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "0"]
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main()
    results[rank] = buf.getvalue()


@pytest.mark.timeout(180)
def test_replica_reductions_two_ranks():
    port = _free_port()
    with mp.Manager() as m:
        res = m.dict()
        mp.start_processes(_rank_main, args=(2, port, res), nprocs=2, start_method="spawn", join=True)
        res = dict(res)
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        assert res[r]["world"] == 2 and res[r]["rank"] == r
        assert res[r]["max"] == 2.0
        assert res[r]["sum"] == 30.0


@pytest.mark.timeout(180)
def test_reference_arm_other_ranks_exit_quietly():
    port = _free_port()
    with mp.Manager() as m:
        res = m.dict()
        mp.start_processes(_reference_rank, args=(2, port, res), nprocs=2, start_method="spawn", join=True)
        res = dict(res)
    assert res[1] == ""  # no JSON line from a non-zero rank
