"""Vocabulary-parallel LM head on one GPU, its ranks emulated in turn.

Each emulated rank runs the records-only kernel on its shard of W with the
shard's index offset; the shards' records, stacked in rank order (padded to
a common count with empty records), go through the multi-rank merge.  The
result must pass the same oracle comparison as the single-call LM head
(indices exact except swaps inside the 1e-3 margin, log-probs within 2e-2),
and must agree with the single call wherever the oracle's lists are free of
near-ties.  No kernel waits on another: the ranks run one after the other."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import check_topk_rows, dev_bf16, exact_ties_free

pytestmark = pytest.mark.gpu


def _sharded(H, W, V, world):
    import block_draft_selection_b200 as bds
    from block_draft_selection_b200.parallel import empty_records, vocab_shard
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    recs = []
    for r in range(world):
        v0, v1 = vocab_shard(V, world, r)
        recs.append(bds.dflash_lmhead_topk_partial(H, W[v0:v1], v_offset=v0, dev_status=status))
    M = H.shape[0]
    P = max(x.shape[1] for x in recs)
    padded = []
    for x in recs:
        if x.shape[1] < P:
            y = empty_records(M, P, x.device)
            y[:, :x.shape[1]] = x
            x = y
        padded.append(x)
    out = bds.dflash_lmhead_topk_merge(torch.stack(padded))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return [t.cpu().numpy() for t in out]


@pytest.mark.parametrize("name,world,nrows", [("tiny", 2, None), ("tiny", 5, None), ("qwen3-4b-bs1", 2, None),
                                              ("qwen3-4b-bs1", 8, None), ("27b-class", 3, 12),
                                              ("qwen3-4b-batched", 2, 16), ("throughput", 4, 16)])
def test_sharded_matches_oracle_and_single(name, world, nrows):
    import block_draft_selection_b200 as bds
    w = syn.workload(name)
    Hb, Wb = syn.hidden(w), syn.lm_head(w)
    H, W = dev_bf16(Hb), dev_bf16(Wb)
    lp, ix, lse = _sharded(H, W, w.V, world)
    lp1, ix1, lse1 = [t.cpu().numpy() for t in bds.dflash_lmhead_topk(H, W)]
    rows = np.arange(w.M)
    if nrows is not None:
        rng = np.random.default_rng(world)
        rows = np.unique(np.concatenate([[0, w.M - 1], rng.choice(w.M, nrows, replace=False)]))
    rlp, rix, rlse, z = oracle.lmhead_topk(Hb[rows], Wb, 16, return_logits=True)
    check_topk_rows(z, rlse, ix, lp, rows=rows)
    assert np.abs(lse[rows] - rlse).max() < 2e-2
    for n, m in enumerate(rows):
        if exact_ties_free(z[n]):
            assert ix[m].tolist() == ix1[m].tolist()
    np.testing.assert_allclose(lse, lse1, rtol=0, atol=1e-4)
    assert (np.diff(lp, axis=1) <= 0).all()


def test_offsets_reach_the_last_shard():
    """A head whose best token lies in the last shard: its index comes back
    shifted by that shard's offset."""
    import block_draft_selection_b200 as bds
    M, V, d = 3, 8000, 256
    rng = np.random.default_rng(4)
    Wf = (rng.standard_normal((V, d)) * 0.05).astype(np.float32)
    Hf = rng.standard_normal((M, d)).astype(np.float32)
    Wf[7777] = Hf[0] * 0.5                       # row 0's clear winner
    H, W = dev_bf16(syn.f32_to_bf16_bits(Hf)), dev_bf16(syn.f32_to_bf16_bits(Wf))
    lp, ix, lse = _sharded(H, W, V, 4)
    assert ix[0, 0] == 7777
