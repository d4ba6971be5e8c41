"""bench.py's multi-rank host logic on CPU with two gloo ranks: per-rank batches,
the max-over-ranks timing reduction, the whole-job aggregate, and that only
rank 0 runs the CPU reference arm."""
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
    import datetime
    import torch.distributed as dist
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import block_draft_synth as syn
        r, lr, ws = bench.dist_env()
        w = syn.workload("tiny")
        wr = bench.rank_workload(w, r)
        h = syn.hidden(wr)
        ms = 10.0 + 5.0 * r                      # rank 1 is the slow one
        ms_max = bench.reduce_max(ms, ws)
        value = bench.aggregate(w.B, ws, ms_max, steps=4)

        class A:                                 # the reference arm's arguments
            steps, warmup, ref_budget_s = 2, 1, 1.0
        ref = bench.reference_arm(A, w)
        dist.barrier()
        q.put((r, lr, ws, int(h[0, 0]), wr.seed, ms_max, value, ref is None))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, l0, w0, h0, s0, m0, v0, none0), (r1, l1, w1, h1, s1, m1, v1, none1) = out
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert s0 != s1 and h0 != h1                 # different blocks per rank
    assert m0 == m1 == 15.0                      # max over ranks
    assert v0 == v1 == pytest.approx(1 * 2 * 4 / 0.015)
    assert not none0 and none1                   # only rank 0 runs the reference arm
