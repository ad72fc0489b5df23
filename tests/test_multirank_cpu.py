"""The benchmark's multi-rank host logic on CPU (gloo, world size 2): every rank
times its own replica; rank 0 reports the maximum time and the summed tokens.
Also checks that a rank which never joins makes the others fail within the
process-group timeout instead of hanging."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    w, r, l = bench.dist_setup(world)
    assert (w, r, l) == (world, rank, rank)
    elapsed = 10.0 + 5.0 * rank      # rank 1 is the slow one
    tokens = 26.0 * (rank + 1)
    ms, tok = bench.aggregate(elapsed, tokens, world, None)
    q.put((rank, ms, tok))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, tok in res:
        assert ms == 15.0  # max over ranks
        assert tok == 26.0 + 52.0  # sum over ranks


def _lonely(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=3))
        q.put("joined")
    except Exception as e:  # the peer never joins: rendezvous must fail, not hang
        q.put(type(e).__name__)


def test_missing_rank_fails_fast():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_lonely, args=(0, 2, _free_port(), q))
    p.start()
    p.join(90)
    assert p.exitcode == 0
    assert q.get(timeout=5) != "joined"


def test_single_rank_aggregate_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(12.5, 26.0, 1) == (12.5, 26.0)


@pytest.mark.parametrize("name", ["decode", "prefill", "wdown", "msweep_M512"])
def test_workloads_are_well_formed(name):
    sys.path.insert(0, ROOT)
    import bench
    cases = bench.workload_cases(name)
    assert cases
    for label, M, N, K, mode, fwht, xk, xdt, outl in cases:
        assert K % 128 == 0 and M >= 1 and N >= 1
        assert mode in ("int8", "int4")
        if fwht:
            assert K & (K - 1) == 0
