"""One draft cycle end to end (LM head -> select -> verify) on the GPU against
the oracle's cycle, on the same seeded inputs: every block of the tiny,
qwen3-4b-bs1, qwen3-4b-batched (tensor-bound 2-CTA orientation) and 27b-class
workloads, and a sample of blocks from every part of the throughput workload
(the GPU runs all 256 blocks; the oracle recomputes the sampled ones).

Target tokens come from the oracle (argmax of the noised hidden state through
W), so both sides verify against the same target.  A block is compared only
where both sides' candidate lists agree exactly on every position (otherwise
a legitimate near-tie swap upstream may change the path)."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16, check_topk_rows

pytestmark = pytest.mark.gpu


def _gpu_cycle(w, H, W, E, M, target):
    import block_draft_selection_b200 as bds
    lp, ix, _ = bds.dflash_lmhead_topk(dev_bf16(H), dev_bf16(W))
    tok, slot, score, _ = bds.dflash_path_select(lp, ix, dev_bf16(E), dev_bf16(M), w.B, w.L)
    acc, nxt = bds.dflash_verify(tok, torch.from_numpy(target.astype(np.int32)).cuda())
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (lp, ix, tok, slot, acc, nxt)]


@pytest.mark.parametrize("wi", [0, 1, 2, 3])
def test_cycle(wi):
    w = syn.workload(wi)
    H, W = syn.hidden(w), syn.lm_head(w)
    E, M = syn.selector_tables(w)
    Hn = syn.target_hidden(w, H)
    target = oracle.argmax_tokens(Hn, W).reshape(w.B, w.L + 1)
    lp, ix, tok, slot, acc, nxt = _gpu_cycle(w, H, W, E, M, target)

    rlp, rix, rlse, z = oracle.lmhead_topk(H, W, 16, return_logits=True)
    check_topk_rows(z, rlse, ix, lp)
    ref = oracle.path_select(rlp, rix, E, M, w.B, w.L)
    racc, rnxt = oracle.verify(ref["path_tok"], target)

    same_lists = (ix.reshape(w.B, w.L, 16) == rix.reshape(w.B, w.L, 16)).all(axis=(1, 2))
    firm = same_lists & (ref["margin"] >= 1e-3)
    assert firm.any()
    np.testing.assert_array_equal(tok[firm], ref["path_tok"][firm])
    np.testing.assert_array_equal(acc[firm], racc[firm])
    np.testing.assert_array_equal(nxt[firm], rnxt[firm])
    # on every block: verification of the GPU's own path is exact
    a2, n2 = oracle.verify(tok, target)
    np.testing.assert_array_equal(acc, a2)
    np.testing.assert_array_equal(nxt, n2)


def test_cycle_sampled_blocks_throughput():
    """Throughput workload (M = 4096 rows in 16 pair tiles of 256): the GPU
    runs the cycle on all 256 blocks; the oracle recomputes the LM head,
    selection and verification of 12 blocks spread over the token tiles
    (the first and last block, one block per 512-row stretch, 2 random)."""
    w = syn.workload(4)
    H, W = syn.hidden(w), syn.lm_head(w)
    E, M = syn.selector_tables(w)
    rng = np.random.default_rng(44)
    blocks = np.unique(np.concatenate([[0, w.B - 1], np.arange(0, w.B, 32) + 7, rng.choice(w.B, 2, replace=False)]))
    rows = (blocks[:, None] * w.L + np.arange(w.L)[None, :]).ravel()
    trows = (blocks[:, None] * (w.L + 1) + np.arange(w.L + 1)[None, :]).ravel()
    Hn = syn.target_hidden(w, H)
    target = np.zeros((w.B, w.L + 1), np.int64)
    target[blocks] = oracle.argmax_tokens(Hn[trows], W).reshape(len(blocks), w.L + 1)
    lp, ix, tok, slot, acc, nxt = _gpu_cycle(w, H, W, E, M, target)

    rlp, rix, rlse, z = oracle.lmhead_topk(H[rows], W, 16, return_logits=True)
    check_topk_rows(z, rlse, ix, lp, rows=rows)
    nb = len(blocks)
    ref = oracle.path_select(rlp, rix, E, M, nb, w.L)
    racc, rnxt = oracle.verify(ref["path_tok"], target[blocks])
    same_lists = (ix[rows].reshape(nb, w.L, 16) == rix.reshape(nb, w.L, 16)).all(axis=(1, 2))
    firm = same_lists & (ref["margin"] >= 1e-3)
    assert firm.any()
    np.testing.assert_array_equal(tok[blocks][firm], ref["path_tok"][firm])
    np.testing.assert_array_equal(acc[blocks][firm], racc[firm])
    np.testing.assert_array_equal(nxt[blocks][firm], rnxt[firm])
    a2, n2 = oracle.verify(tok[blocks], target[blocks])
    np.testing.assert_array_equal(acc[blocks], a2)
    np.testing.assert_array_equal(nxt[blocks], n2)
