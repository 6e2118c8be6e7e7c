"""The N > 1 host path of bench.py on CPU: two processes over gloo (no GPU).

bench.py runs one independent call per rank (no collective on the data path);
the process group carries only the barriers and the max over ranks of the
timings. These tests start 2 ranks with the spawn method and check the
barrier, the max over ranks, that ranks draw different inputs of the same
shape, and that the reference arm runs on rank 0 only.
"""

import contextlib
import io
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import synthetic as S
    dist, r, w, _ = bench._dist_setup(world, backend="gloo")
    bench._barrier(dist)
    m = bench._max_over_ranks(dist, 10.0 + 3.0 * r, device="cpu")
    wl = bench.replica_workload(S.WORKLOADS["tiny"], r)
    q, _, _ = S.make_qkv(wl)
    bench._barrier(dist)
    dist.destroy_process_group()
    out.put((r, w, m, wl.seed, tuple(q.shape), float(q.double().sum())))


def test_two_ranks_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == world for r in res)
    assert all(r[2] == 13.0 for r in res)                     # max over ranks reaches every rank
    assert res[0][3] != res[1][3] and res[0][4] == res[1][4]  # own seed, same shape
    assert res[0][5] != res[1][5]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert rc == 0 and buf.getvalue() == ""
