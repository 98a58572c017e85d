"""Host logic of the multi-GPU path on CPU: two gloo ranks run bench.py's
distributed context (barrier, max over ranks, replica seeds, whole-job rate)
and a rank that leaves early makes the other's collective fail within the
process group's timeout instead of hanging. The path shards by replicas, so
there is no data-path collective to test."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    try:
        ctx = bench.Ctx(backend="gloo", timeout_s=5.0)
        if mode == "leave" and rank == 1:
            out.put((rank, "left"))
            return  # leaves between steps, before the collective
        ctx.barrier()
        ms = ctx.max_over_ranks(1.0 + rank)
        seed = bench.replica_seed(2, rank)
        ctx.barrier()
        ctx.close()
        out.put((rank, ("ok", ms, seed)))
    except Exception as e:  # noqa: BLE001 - reported to the parent
        out.put((rank, ("error", type(e).__name__)))


def _run(mode, world=2, timeout=60):
    ctxm = mp.get_context("spawn")
    out = ctxm.Queue()
    port = _free_port()
    procs = [ctxm.Process(target=_worker, args=(r, world, port, mode, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=timeout) for _ in procs)
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
    return res


def test_two_replicas_max_over_ranks_and_seeds():
    import bench
    res = _run("normal")
    assert res[0][0] == "ok" and res[1][0] == "ok", res
    assert res[0][1] == res[1][1] == 2.0  # every rank sees the slowest rank's time
    assert res[0][2] != res[1][2]         # each replica draws its own inputs
    # whole-job rate: both ranks' units over the slowest rank's time
    assert bench.whole_job_rate(2, 32768, 2.0) == pytest.approx(2 * 32768 / 2e-3)


def test_rank_leaving_fails_the_others_collective():
    res = _run("leave")
    assert res[1] == "left"
    assert res[0][0] == "error", res
