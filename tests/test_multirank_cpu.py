"""The bench's multi-rank plumbing on CPU with the gloo backend, world size 2:
replicas draw distinct batches, the timing is the max over ranks, and the
reference arm runs on rank 0 only."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist

    try:
        r, w = bench.dist_init("gloo", timeout_s=60)
        got = bench.max_over_ranks([1.0 + r, 10.0 - r, 3.5])
        bench.barrier()
        seed = bench.rank_seed(0, r)
        ref_rc = bench.run_reference(type("A", (), {})()) if r == 1 else None
        q.put((r, w, got, seed, ref_rc))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_max_and_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, g0, s0, _), (r1, w1, g1, s1, ref1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert g0 == g1 == [2.0, 10.0, 3.5]          # element-wise max over both ranks
    assert s0 != s1                               # each replica draws its own batch
    assert ref1 == 0                              # reference arm: non-zero ranks exit without work


def test_single_rank_max_is_identity(monkeypatch):
    import bench

    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
