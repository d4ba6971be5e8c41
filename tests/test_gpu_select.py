"""Pair scores + max-sum walk on the GPU against the oracle.

Both sides get the same seeded candidate lists, so a near-tie upstream cannot
hide a selector bug.  Pair scores must lie within an a priori fp32 error bound
of the exact ones; the selected path must equal the oracle's wherever the
oracle's margin (best minus second-best path score) is at least 1e-3."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _run(logp, idx, E, M, B, L, pair=True):
    import block_draft_selection_b200 as bds
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, slot, score, S = bds.dflash_path_select(
        torch.from_numpy(logp).cuda(), torch.from_numpy(idx).cuda(), dev_bf16(E), dev_bf16(M), B, L,
        pair_scores=pair, dev_status=status)
    torch.cuda.synchronize()
    return (tok.cpu().numpy(), slot.cpu().numpy(), score.cpu().numpy(),
            None if S is None else S.cpu().numpy(), int(status.item()))


def _pair_bound(logp, idx, E, M, B, L):
    """|fp32 S - exact S| <= (2r+4) u (|lp_j| + |lp_k| + |e_a| |M| |e_b|):
    bf16 products are exact in fp32; u = e.M and u.e each accumulate r terms."""
    r = M.shape[0]
    absb = lambda b: b & np.uint16(0x7FFF)       # |x| of a bf16 bit pattern
    A = oracle.pair_scores(np.abs(logp), idx, absb(E), absb(M), B, L)
    return (2 * r + 4) * U * A + 1e-7, A


def _check(logp, idx, E, M, B, L):
    tok, slot, score, S, status = _run(logp, idx, E, M, B, L)
    assert status == 0
    ref = oracle.path_select(logp, idx, E, M, B, L)
    if L == 1:           # no pairs: every path scores 0, the tie rule picks slot 0
        assert (slot == 0).all() and (score == 0).all()
        assert (tok[:, 0] == idx[:, 0]).all()
        return None
    if L > 1:
        bound, A = _pair_bound(logp, idx, E, M, B, L)
        err = np.abs(S - ref["pair_scores"])
        assert (err <= bound).all(), (err - bound).max()
    firm = ref["margin"] >= 1e-3
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])
    np.testing.assert_array_equal(tok[firm], ref["path_tok"][firm])
    # every returned path is a valid path through the lists
    for b in range(B):
        for i in range(L):
            assert tok[b, i] == idx[b * L + i, slot[b, i]]
    if L > 1:
        pb = np.array([sum(bound[b, i, ref["path_slot"][b, i], ref["path_slot"][b, i + 1]] +
                           (L - 1) * 2 * U * A[b, i, ref["path_slot"][b, i], ref["path_slot"][b, i + 1]]
                           for i in range(L - 1)) for b in range(B)])
        np.testing.assert_array_less(np.abs(score[firm] - ref["path_score"][firm]), pb[firm] + 1e-6)
    return firm


@pytest.mark.parametrize("wi", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("scale", [1.0, 0.3, 3.0])
def test_workload_shapes(wi, scale):
    w = syn.workload(wi)
    logp, idx = syn.synthetic_topk(w.B, w.L, w.V, w.seed + 100)
    E, M = syn.selector_tables(w, scale)
    _check(logp, idx, E, M, w.B, w.L)


@pytest.mark.parametrize("B,L,r", [(3, 1, 8), (2, 2, 8), (7, 3, 16), (5, 16, 8), (4, 16, 128), (300, 9, 24)])
def test_edge_shapes(B, L, r):
    V = 3000
    logp, idx = syn.synthetic_topk(B, L, V, B + L + r)
    rng = syn.rng_for(r, "E")
    E = syn.f32_to_bf16_bits(rng.standard_normal((V, r)).astype(np.float32) * 0.4)
    M = syn.f32_to_bf16_bits(rng.standard_normal((r, r)).astype(np.float32) * 0.4)
    _check(logp, idx, E, M, B, L)


def test_hand_case(golden):
    g = golden("viterbi_hand.json")
    B, L, V, r = g["B"], g["L"], g["V"], g["r"]
    logp = np.tile(-np.arange(16, dtype=np.float32), (B * L, 1))
    idx = np.array([[100 * i + j for j in range(16)] for i in range(L)], dtype=np.int32)
    E = np.zeros((V, r), np.float32)
    for v, s, x in g["E_nonzero"]:
        E[v, s] = x
    M = np.zeros((r, r), np.float32)
    for s, t, x in g["M_nonzero"]:
        M[s, t] = x
    tok, slot, score, _, status = _run(logp, idx, syn.f32_to_bf16_bits(E), syn.f32_to_bf16_bits(M), B, L)
    assert status == 0
    assert slot[0].tolist() == g["path_slot"]
    assert tok[0].tolist() == g["path_tok"]
    assert score[0] == g["path_score"]


def test_zero_pair_term_is_top1():
    B, L, V, r = 9, 7, 1000, 16
    logp, idx = syn.synthetic_topk(B, L, V, 77)
    E = np.zeros((V, r), np.uint16)
    M = syn.f32_to_bf16_bits(np.ones((r, r), np.float32))
    tok, slot, score, _, _ = _run(logp, idx, E, M, B, L)
    assert (slot == 0).all()
    assert (tok == idx.reshape(B, L, 16)[:, :, 0]).all()


def test_bad_index_is_reported():
    B, L, V, r = 2, 4, 100, 8
    logp, idx = syn.synthetic_topk(B, L, V, 5)
    idx = idx.copy()
    idx[3, 7] = V + 5
    E, M = syn.selector_tables(syn.Workload("t", B, L, L, 8, V, r, 0.3, 0), 1.0)
    *_, status = _run(logp, idx, E, M, B, L, pair=False)
    assert status == 6


@pytest.mark.parametrize("wi", [0, 1, 2, 3, 4])
def test_select_verify_matches_separate_calls(wi):
    """The fused selector+verifier gives bit-identical paths to the selector
    alone, and, wherever the oracle's path is firm, the oracle's verification
    of that path.  Targets are the oracle's path, corrupted per position with
    probability 0.3."""
    import block_draft_selection_b200 as bds
    w = syn.workload(wi)
    logp, idx = syn.synthetic_topk(w.B, w.L, w.V, w.seed + 200)
    E, M = syn.selector_tables(w)
    ref = oracle.path_select(logp, idx, E, M, w.B, w.L)
    rng = np.random.default_rng(wi)
    t = ref["path_tok"].astype(np.int64)
    corrupt = rng.random(t.shape) < 0.3
    t = np.where(corrupt, (t + 1) % w.V, t)
    target = np.concatenate([t, rng.integers(0, w.V, (w.B, 1))], axis=1).astype(np.int32)
    lp_d, ix_d = torch.from_numpy(logp).cuda(), torch.from_numpy(idx).cuda()
    E_d, M_d = dev_bf16(E), dev_bf16(M)
    tok, slot, score, _ = bds.dflash_path_select(lp_d, ix_d, E_d, M_d, w.B, w.L)
    t_d = torch.from_numpy(target).cuda()
    tok2, slot2, score2, acc, nxt = bds.dflash_select_verify(lp_d, ix_d, E_d, M_d, t_d, w.B, w.L)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(tok2.cpu().numpy(), tok.cpu().numpy())
    np.testing.assert_array_equal(slot2.cpu().numpy(), slot.cpu().numpy())
    np.testing.assert_array_equal(score2.cpu().numpy(), score.cpu().numpy())
    racc, rnxt = oracle.verify(ref["path_tok"], target)
    firm = ref["margin"] >= 1e-3 if w.L > 1 else np.ones(w.B, bool)
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(acc.cpu().numpy()[firm], racc[firm])
    np.testing.assert_array_equal(nxt.cpu().numpy()[firm], rnxt[firm])
