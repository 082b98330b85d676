"""The multi-process side of bench.py on the CPU: two ranks over gloo
(127.0.0.1). bench.py runs one independent replica per GPU (the GEMV has no
exchange step), so what has to hold across ranks is the timing plumbing: the
barrier, the max of the ranks' device times, the sum of their bytes, the
whole-job figure built from them, and the reference arm running on rank 0
only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    try:
        import bench
        d = bench.Dist()
        d.init("gloo")
        d.barrier()
        mx = d.max(1.5 + rank)            # rank 1 is the slow one
        sm = d.sum(10.0 * (rank + 1))
        value, ms = bench.whole_job(1e9 * (rank + 1), 2.0 + rank, d)
        d.barrier()
        # the reference arm: rank 0 alone would run it; other ranks return 0 at once
        called = []
        orig = bench.run_reference
        bench.run_reference = lambda args, dist: called.append(dist.rank) or {"impl": "reference"}
        try:
            rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "3",
                             "--warmup", "3"])
        finally:
            bench.run_reference = orig
        d.close()
        q.put((rank, mx, sm, value, ms, rc, called))
    except Exception as e:  # reported to the parent
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_timing_plumbing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res = {r[0]: r for r in out}
    for r in range(world):
        assert res[r][1] != "error", res[r]
        _, mx, sm, value, ms, rc, called = res[r]
        assert mx == 2.5 and sm == 30.0               # max / sum over the ranks
        assert ms == 3.0                               # the slowest rank's time
        assert value == pytest.approx(3e9 / 3e-3 / 1e9)  # all ranks' bytes / max time
        assert rc == 0
        assert called == ([0] if r == 0 else [])      # reference arm on rank 0 only
