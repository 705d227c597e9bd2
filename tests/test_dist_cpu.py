"""The benchmark's multi-process plumbing on CPU: two gloo ranks, launched
like torchrun's (RANK / WORLD_SIZE / MASTER_* in the environment), take the
same collective steps; the timed value is the max over ranks, and the
whole-job throughput of the replicas counts every rank's units."""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("lbq_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "LBQ_DIST_BACKEND": "gloo"})
    bench = _bench()
    d = bench.Dist()
    d.barrier()
    # each rank "measured" a different time; the job's time is the slowest
    ms = [3.0, 7.5][rank]
    m = d.max(ms)
    d.barrier()
    out[rank] = (d.world, d.rank, m, bench.replica_value(1e9, d.world, m))
    d.close()


def test_two_gloo_ranks_max_and_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        w, rk, m, v = out[r]
        assert (w, rk) == (world, r)
        assert m == 7.5
        assert v == pytest.approx(1e9 * 2 / 7.5e-3 / 1e9)


def test_replica_value_single_rank():
    bench = _bench()
    assert bench.replica_value(2e9, 1, 1000.0) == pytest.approx(2.0)
