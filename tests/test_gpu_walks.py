"""Walks from the last verified token and rejection-sampling verification on
the GPU against the oracle.

Greedy: the path must equal the oracle's wherever every step's margin (chosen
minus runner-up score, in the oracle) is at least 1e-3 -- past an ambiguous
step the two walks may legitimately part.  Sampling: the path must equal the
oracle's wherever every draw's uniform is at least 1e-4 from a cumulative
boundary; the reported distributions must agree to 1e-5.  Rejection
sampling: accept lengths must equal the oracle's wherever every tested
position is decided by more than 1e-6 (relative), and the drawn token
wherever the scaled uniform is more than 1e-7 (of the total) from a boundary;
elsewhere the GPU's token must be a valid draw for a uniform within 1e-6.
The kernel evaluates every deciding probability with fp64 exponentials of
fp32 logits; 1e-6 covers its fp32 per-slice sums (8192 terms each)."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16

pytestmark = pytest.mark.gpu


def _tables(seed, V, r, scale=0.5):
    rng = syn.rng_for(seed, "E")
    E = syn.f32_to_bf16_bits(rng.standard_normal((V, r)).astype(np.float32) * scale)
    M = syn.f32_to_bf16_bits(rng.standard_normal((r, r)).astype(np.float32) * scale)
    return E, M


def _walk(logp, idx, E, M, anchor, B, L, u=None, T=1.0, target=None):
    import block_draft_selection_b200 as bds
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = bds.dflash_path_walk(torch.from_numpy(logp).cuda(), torch.from_numpy(idx).cuda(), dev_bf16(E),
                               dev_bf16(M), torch.from_numpy(anchor).cuda(), B, L,
                               uniforms=None if u is None else torch.from_numpy(u).cuda(), temperature=T,
                               target=None if target is None else torch.from_numpy(target).cuda(),
                               dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return [None if t is None else t.cpu().numpy() for t in out]


WALK_SHAPES = [(1, 7, 151936, 64), (16, 5, 151936, 64), (200, 4, 5000, 32), (3, 16, 3000, 128),
               (2, 1, 1000, 16), (40, 12, 20000, 64), (256, 16, 129280, 128)]


@pytest.mark.parametrize("B,L,V,r", WALK_SHAPES)
def test_greedy_walk(B, L, V, r):
    seed = B + L + r
    logp, idx = syn.synthetic_topk(B, L, V, seed)
    E, M = _tables(seed, V, r)
    anchor = syn.anchors(B, V, seed)
    tok, slot, score, q, _, _ = _walk(logp, idx, E, M, anchor, B, L)
    assert q is None
    ref = oracle.greedy_walk(logp, idx, E, M, anchor, B, L)
    firm = (ref["margin"] >= 1e-3).all(axis=1)
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])
    np.testing.assert_array_equal(tok[firm], ref["path_tok"][firm])
    np.testing.assert_allclose(score[firm], ref["path_score"][firm], rtol=1e-5, atol=1e-4)
    idx3 = idx.reshape(B, L, 16)
    assert ((slot >= 0) & (slot < 16)).all()
    assert (np.take_along_axis(idx3, slot[:, :, None], axis=2)[:, :, 0] == tok).all()


def test_greedy_walk_hand_case(golden):
    g = golden("walks_hand.json")["greedy"]
    B, L, V, r = g["B"], g["L"], g["V"], g["r"]
    logp = np.tile(-np.arange(16, dtype=np.float32), (B * L, 1))
    idx = np.array([[100 * i + j for j in range(16)] for i in range(L)], dtype=np.int32)
    E = np.zeros((V, r), np.float32)
    for v, s, x in g["E_nonzero"]:
        E[v, s] = x
    M = np.zeros((r, r), np.float32)
    for s, t, x in g["M_nonzero"]:
        M[s, t] = x
    tok, slot, score, *_ = _walk(logp, idx, syn.f32_to_bf16_bits(E), syn.f32_to_bf16_bits(M),
                                 np.array([g["anchor"]], np.int32), B, L)
    assert slot[0].tolist() == g["path_slot"]
    assert tok[0].tolist() == g["path_tok"]
    assert score[0] == g["path_score"]


def test_greedy_walk_with_verification():
    B, L, V, r = 64, 7, 151936, 64
    logp, idx = syn.synthetic_topk(B, L, V, 5)
    E, M = _tables(5, V, r)
    anchor = syn.anchors(B, V, 5)
    ref = oracle.greedy_walk(logp, idx, E, M, anchor, B, L)
    rng = np.random.default_rng(5)
    t = np.where(rng.random((B, L)) < 0.25, (ref["path_tok"] + 1) % V, ref["path_tok"])
    target = np.concatenate([t, rng.integers(0, V, (B, 1))], axis=1).astype(np.int32)
    tok, slot, score, q, acc, nxt = _walk(logp, idx, E, M, anchor, B, L, target=target)
    firm = (ref["margin"] >= 1e-3).all(axis=1)
    racc, rnxt = oracle.verify(ref["path_tok"], target)
    np.testing.assert_array_equal(acc[firm], racc[firm])
    np.testing.assert_array_equal(nxt[firm], rnxt[firm])


@pytest.mark.parametrize("T", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("B,L,V,r", WALK_SHAPES)
def test_sample_walk(B, L, V, r, T):
    seed = 3 * B + L
    logp, idx = syn.synthetic_topk(B, L, V, seed, spread=0.5)
    E, M = _tables(seed, V, r, 0.3)
    anchor = syn.anchors(B, V, seed)
    u = syn.uniforms((B, L), seed, "u_walk")
    tok, slot, score, q, _, _ = _walk(logp, idx, E, M, anchor, B, L, u=u, T=T)
    ref = oracle.sample_walk(logp, idx, E, M, anchor, u, T, B, L)
    firm = (ref["gap"] >= 1e-4).all(axis=1)
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])
    np.testing.assert_array_equal(tok[firm], ref["path_tok"][firm])
    np.testing.assert_allclose(q[firm], ref["q"][firm], rtol=0, atol=1e-5)
    np.testing.assert_allclose(q.sum(axis=2), 1.0, atol=1e-5)
    idx3 = idx.reshape(B, L, 16)
    assert (np.take_along_axis(idx3, slot[:, :, None], axis=2)[:, :, 0] == tok).all()


def _verify_inputs(B, L, V, seed, T, spread=0.5):
    """A sampled draft (the oracle's walk) and target logits where each draft
    token's logit is raised by a random amount around the level at which the
    target's p(x) matches a typical draft q(x), so that acceptance happens at
    a spread of rates.  The logits are N(0, 2^2): the partition sum is about
    V exp(2 / T^2), so p(x) ~ 1 needs a raise of about T ln V + 2 / T."""
    logp, idx = syn.synthetic_topk(B, L, V, seed, spread=0.5)
    E, M = _tables(seed, V, 32, 0.3)
    anchor = syn.anchors(B, V, seed)
    u = syn.uniforms((B, L), seed, "u_walk")
    w = oracle.sample_walk(logp, idx, E, M, anchor, u, T, B, L)
    z = syn.target_logits(B * (L + 1), V, seed)
    crit = T * np.log(V) + 2.0 / T
    bump = syn.rng_for(seed, "gate").uniform(crit * (1 - spread), crit * (1 + spread), size=(B, L))
    bump = bump.astype(np.float32)
    z3 = z.reshape(B, L + 1, V)
    for b in range(B):
        for i in range(L):
            z3[b, i, w["path_tok"][b, i]] += bump[b, i]
    ua = syn.uniforms((B, L), seed, "u_accept")
    ur = syn.uniforms((B,), seed, "u_resample")
    return dict(z=z, draft=w["path_tok"].astype(np.int32), slot=w["path_slot"].astype(np.int32), idx=idx,
                q=w["q"].astype(np.float32), ua=ua, ur=ur)


def _run_rejection(d, T):
    import block_draft_selection_b200 as bds
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    acc, nxt = bds.dflash_verify_rejection(t(d["z"]), T, t(d["draft"]), t(d["slot"]), t(d["idx"]), t(d["q"]),
                                           t(d["ua"]), t(d["ur"]), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return acc.cpu().numpy(), nxt.cpu().numpy()


def _valid_draw(res, u, v, tol):
    """v is the inverse-CDF draw of `res` for some uniform within tol of u."""
    c = np.cumsum(res)
    t = u * c[-1]
    lo = c[v - 1] if v > 0 else 0.0
    return res[v] > 0 and lo <= t + tol * c[-1] and c[v] >= t - tol * c[-1]


@pytest.mark.parametrize("B,L,V,T", [(1, 7, 151936, 1.0), (64, 7, 151936, 0.7), (16, 5, 151936, 1.5), (2, 31, 9000, 1.0),
                                     (8, 4, 4096, 1.0), (5, 3, 8193, 1.0), (9, 6, 10001, 1.0),
                                     (3, 16, 20000, 2.0), (32, 1, 30000, 1.0)])
def test_verify_rejection(B, L, V, T):
    d = _verify_inputs(B, L, V, 11 * B + L, T)
    acc, nxt = _run_rejection(d, T)
    p = oracle.target_probs(d["z"], T).reshape(B, L + 1, V)
    ref = oracle.verify_rejection(d["draft"], d["slot"], d["idx"], d["q"], p, d["ua"], d["ur"])
    assert ((acc >= 1) & (acc <= L + 1)).all()
    # decided acceptance: every tested position far from its threshold
    am = ref["accept_margin"]
    tested = np.arange(L)[None, :] < np.minimum(ref["accept_len"], L)[:, None]
    firm_acc = np.where(tested, am > 1e-6, True).all(axis=1)
    assert firm_acc.mean() > 0.9
    np.testing.assert_array_equal(acc[firm_acc], ref["accept_len"][firm_acc])
    firm_tok = firm_acc & (ref["resample_margin"] > 1e-7)
    np.testing.assert_array_equal(nxt[firm_tok], ref["next_token"][firm_tok])
    # everywhere the accept length agrees, the drawn token is a valid draw
    cand = d["idx"].reshape(B, L, 16)
    for b in np.nonzero(acc == ref["accept_len"])[0]:
        n = acc[b] - 1
        if n == L:
            res = p[b, L]
        else:
            qv = np.zeros(V)
            qv[cand[b, n]] = d["q"][b, n]
            res = np.maximum(0.0, p[b, n] - qv)
        assert _valid_draw(res, float(d["ur"][b]), int(nxt[b]), 1e-6), (b, nxt[b], ref["next_token"][b])
    # both outcomes occur in these inputs
    assert (acc < L + 1).any() and (acc > 1).any() or L == 1


def test_verify_rejection_all_accepted_draws_bonus():
    """u_accept = 0 accepts every draft with p > 0: the next token is p_L's draw."""
    B, L, V, T = 6, 5, 20000, 1.0
    d = _verify_inputs(B, L, V, 3, T)
    d["ua"] = np.zeros((B, L), np.float32)
    acc, nxt = _run_rejection(d, T)
    assert (acc == L + 1).all()
    p = oracle.target_probs(d["z"], T).reshape(B, L + 1, V)
    for b in range(B):
        assert _valid_draw(p[b, L], float(d["ur"][b]), int(nxt[b]), 1e-6)


def test_verify_rejection_never_resamples_rejected_token():
    B, L, V, T = 128, 4, 20000, 1.0
    d = _verify_inputs(B, L, V, 4, T, spread=0.9)
    acc, nxt = _run_rejection(d, T)
    rej = acc <= L
    assert rej.any()
    n = acc[rej] - 1
    assert (nxt[rej] != d["draft"][rej, n]).all()


def test_verify_rejection_bad_index_is_reported():
    import block_draft_selection_b200 as bds
    B, L, V, T = 2, 3, 5000, 1.0
    d = _verify_inputs(B, L, V, 6, T)
    d["draft"] = d["draft"].copy()
    d["draft"][1, 0] = V + 3
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bds.dflash_verify_rejection(t(d["z"]), T, t(d["draft"]), t(d["slot"]), t(d["idx"]), t(d["q"]),
                                t(d["ua"]), t(d["ur"]), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6


def test_verify_rejection_workspace_reuse_and_masked_slices():
    """One workspace over several calls of different batch sizes gives the
    results of a fresh workspace each time.  Rows whose logits are -inf
    outside a few slices (whole slices without mass, a slice with mass in its
    first 232 entries only) still give valid draws."""
    import block_draft_selection_b200 as bds
    L, V, T = 5, 40000, 1.0
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Bmax = 12
    n_ws = bds.dflash_verify_rejection_workspace(Bmax, L, V)
    ws = torch.full((n_ws,), 0xAB, dtype=torch.uint8, device="cuda")    # no initial contents needed
    for B, seed in ((Bmax, 21), (3, 22), (Bmax, 21), (7, 23)):
        d = _verify_inputs(B, L, V, seed, T)
        z = d["z"].reshape(B, L + 1, V)
        if seed == 23:
            # every row keeps mass only in [8192, 16384) and [32768, 33000) (the drafts' raised logits aside)
            keep = np.zeros(V, bool)
            keep[8192:16384] = True
            keep[32768:33000] = True
            cand = d["idx"].reshape(B, L, 16)
            for b in range(B):
                for i in range(L + 1):
                    m = keep.copy()
                    if i < L:
                        m[cand[b, i]] = True
                    z[b, i, ~m] = -np.inf
        d["z"] = z.reshape(B * (L + 1), V)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        args = (t(d["z"]), T, t(d["draft"]), t(d["slot"]), t(d["idx"]), t(d["q"]), t(d["ua"]), t(d["ur"]))
        acc, nxt = bds.dflash_verify_rejection(*args, ws=ws, dev_status=status)
        acc2, nxt2 = bds.dflash_verify_rejection(*args, dev_status=status)     # a fresh workspace
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        np.testing.assert_array_equal(acc.cpu().numpy(), acc2.cpu().numpy())
        np.testing.assert_array_equal(nxt.cpu().numpy(), nxt2.cpu().numpy())
        acc, nxt = acc.cpu().numpy(), nxt.cpu().numpy()
        p = oracle.target_probs(d["z"], T).reshape(B, L + 1, V)
        cand = d["idx"].reshape(B, L, 16)
        for b in range(B):
            n = acc[b] - 1
            if n == L:
                res = p[b, L]
            else:
                qv = np.zeros(V)
                qv[cand[b, n]] = d["q"][b, n]
                res = np.maximum(0.0, p[b, n] - qv)
            assert _valid_draw(res, float(d["ur"][b]), int(nxt[b]), 1e-6), (B, seed, b, nxt[b])
