"""The vocabulary-parallel LM head's rank logic on CPU with gloo ranks.

Each rank's record producer and the merge are stand-ins written here from
the oracle (one record per row per shard: the shard's max, sum of
exponentials and top-16, indices shifted to the full vocabulary); the code
under test is the orchestration in block_draft_selection_b200.parallel --
the shard plan, the index offsets, the padding to a common record count and
the rank-ordered all-gather.  The result must equal the oracle's top-16 of
the whole head."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

K = 16


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _records_from_oracle(H_bits, W_bits, v0, n_records):
    """Stand-in producer: the shard's logits from the oracle, split into
    n_records contiguous column groups, one record each."""
    import oracle
    z = oracle.logits(H_bits, W_bits)                       # [M, Vs] float64
    M, Vs = z.shape
    out = np.zeros((M, n_records, 36), np.float32)
    bounds = np.linspace(0, Vs, n_records + 1).astype(int)
    for r in range(n_records):
        zz = z[:, bounds[r]:bounds[r + 1]]
        m = zz.max(axis=1)
        s = np.exp(zz - m[:, None]).sum(axis=1)
        order = np.lexsort((np.arange(zz.shape[1])[None, :].repeat(M, 0), -zz), axis=1)[:, :K]
        out[:, r, 0], out[:, r, 1] = m, s
        out[:, r, 4:20] = np.take_along_axis(zz, order, axis=1)
        out[:, r, 20:36] = (order + bounds[r] + v0).astype(np.int32).view(np.float32)
    return torch.from_numpy(out)


def _merge_from_oracle(records):
    """Stand-in merge: the union's top-16 (value desc, index asc) and lse."""
    rec = records.numpy()
    W_, M, P, _ = rec.shape
    rec = rec.transpose(1, 0, 2, 3).reshape(M, W_ * P, 36)
    m, s = rec[:, :, 0].astype(np.float64), rec[:, :, 1].astype(np.float64)
    ok = np.isfinite(m)
    mm = np.where(ok, m, -np.inf).max(axis=1)
    lse = mm + np.log(np.where(ok, s * np.exp(np.where(ok, m, 0) - mm[:, None]), 0).sum(axis=1))
    vals = rec[:, :, 4:20].reshape(M, -1).astype(np.float64)
    idx = rec[:, :, 20:36].copy().view(np.int32).reshape(M, -1)
    valid = idx != 0x7FFFFFFF
    lp = np.zeros((M, K))
    ix = np.zeros((M, K), np.int64)
    for row in range(M):
        v, i = vals[row][valid[row]], idx[row][valid[row]]
        o = np.lexsort((i, -v))[:K]
        lp[row], ix[row] = v[o] - lse[row], i[o]
    return torch.from_numpy(lp), torch.from_numpy(ix), torch.from_numpy(lse)


def _worker(rank, world, port, q, V, n_rec_by_rank):
    import datetime
    import torch.distributed as dist
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import block_draft_synth as syn
        from block_draft_selection_b200.parallel import VocabParallelLMHead, vocab_shard
        w = syn.Workload("vp", B=2, L=3, P=4, d=64, V=V, r=8, sigma=0.3, seed=11)
        H, W = syn.hidden(w), syn.lm_head(w)
        v0, v1 = vocab_shard(V, world, rank)
        head = VocabParallelLMHead(W[v0:v1], v0,
                                   partial_fn=lambda h, ws, off: _records_from_oracle(h, ws, off, n_rec_by_rank[rank]),
                                   merge_fn=_merge_from_oracle)
        lp, ix, lse = head(H)
        q.put((rank, v0, v1, lp.numpy(), ix.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,V,n_rec", [(2, 1000, (3, 3)), (2, 777, (2, 5)), (3, 1601, (1, 4, 2))])
def test_vocab_parallel_ranks(world, V, n_rec):
    import oracle
    import block_draft_synth as syn
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, V, n_rec)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=120) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the shards tile [0, V) in rank order, aligned to 16 rows
    assert out[0][1] == 0 and out[-1][2] == V
    for a, b in zip(out, out[1:]):
        assert a[2] == b[1] and a[2] % 16 == 0
    w = syn.Workload("vp", B=2, L=3, P=4, d=64, V=V, r=8, sigma=0.3, seed=11)
    rlp, rix, rlse = oracle.lmhead_topk(syn.hidden(w), syn.lm_head(w), K)
    for _, _, _, lp, ix, lse in out:           # every rank holds the full result
        np.testing.assert_array_equal(ix, rix)
        np.testing.assert_allclose(lp, rlp, rtol=0, atol=1e-5)
        np.testing.assert_allclose(lse, rlse, rtol=0, atol=1e-5)


def test_vocab_shard_plan():
    from block_draft_selection_b200.parallel import vocab_shard
    for V in (16, 17, 4096, 151936, 129280, 100):
        for world in (1, 2, 3, 8):
            shards = [vocab_shard(V, world, r) for r in range(world)]
            assert shards[0][0] == 0 and shards[-1][1] == V
            assert all(a[1] == b[0] for a, b in zip(shards, shards[1:]))
            assert all(s[0] % 16 == 0 for s in shards)
            sizes = [s[1] - s[0] for s in shards]
            assert max(sizes) - min(sizes) <= 16 + (V % 16 != 0) * 16
