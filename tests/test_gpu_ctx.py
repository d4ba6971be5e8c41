"""The pages' context-gated pair scorer on the GPU against the oracle.

Scores: every table entry within an a priori bound of the oracle's fp64
value (the token tables A, B for the whole vocabulary and the gate are
fp32-accumulated GEMMs of exact bf16 products;
the gate's sigmoid and the e-term dot product add fp32 roundings).  Walks:
the path must equal the oracle's where the oracle's margin allows it --
max-sum: best minus second-best path score >= 1e-3; greedy: every step's
chosen-minus-runner-up >= 1e-3; sampled: every uniform >= 1e-4 from a
cumulative boundary (and the reported distributions within 1e-5)."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _inputs(w, e, seed_off=0):
    Emb = syn.lm_head(w)                                   # tied embedding table
    H = syn.hidden(w)
    Pab, Pg = syn.ctx_scorer_weights(w, e)
    logp, idx = syn.synthetic_topk(w.B, w.L, w.V, w.seed + 300 + seed_off, spread=0.5)
    anchor = syn.anchors(w.B, w.V, w.seed + seed_off)
    return Emb, H, Pab, Pg, logp, idx, anchor


def _run(Emb, H, Pab, Pg, logp, idx, anchor, B, L, V, walk="maxsum", u=None, T=1.0, target=None):
    import block_draft_selection_b200 as bds
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tab = bds.dflash_ctx_table(dev_bf16(Emb), dev_bf16(Pab))
    gate = bds.dflash_ctx_gate(dev_bf16(H), dev_bf16(Pg))
    out = bds.dflash_ctx_walk(t(logp), t(idx), t(anchor), tab, gate, B, L, V, walk=walk,
                              uniforms=None if u is None else t(u), temperature=T, want_tables=True,
                              target=None if target is None else t(target), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return [None if x is None else x.cpu().numpy() for x in out]


def _table_bound(Emb, H, Pab, Pg, logp, idx, anchor, B, L):
    """A priori bound on |GPU table - exact table| per entry."""
    from block_draft_synth import bf16_bits_to_f32
    f = lambda b: bf16_bits_to_f32(b).astype(np.float64)
    Pabf = f(Pab)
    e = Pabf.shape[0] // 2
    Pa, Pb = Pabf[:e], Pabf[e:]
    d = Pabf.shape[1]
    idx3 = np.asarray(idx, np.int64).reshape(B, L, 16)
    cand = f(Emb[idx3])                                   # [B, L, 16, d]
    anc = f(Emb[np.asarray(anchor, np.int64)])            # [B, d]
    gemm_err = lambda x, w: 4 * d * 2.0 ** -23 * (np.abs(x) @ np.abs(w).T) + 1e-6
    A, dA = cand @ Pa.T, gemm_err(cand, Pa)
    Bv, dB = cand @ Pb.T, gemm_err(cand, Pb)
    Aa, dAa = anc @ Pa.T, gemm_err(anc, Pa)
    Hf = f(H).reshape(B, L, d)
    Pgf = f(Pg)
    g = oracle.ctx_scorer.sigmoid(Hf @ Pgf.T)             # [B, L, e]
    dg = 0.25 * gemm_err(Hf, Pgf) + 4 * U
    bound = np.empty((B, L, 16, 16))
    for t in range(L):
        pa = np.repeat(np.abs(Aa)[:, None, :], 16, axis=1) if t == 0 else np.abs(A[:, t - 1])
        pda = np.repeat(dAa[:, None, :], 16, axis=1) if t == 0 else dA[:, t - 1]
        gt, dgt = g[:, t][:, None, :], dg[:, t][:, None, :]
        bb, dbb = np.abs(Bv[:, t]), dB[:, t]
        term = lambda x, y: np.einsum("bjq,bkq->bjk", x, y)
        prod = term(pa * gt, bb)
        bound[:, t] = (term(pda * gt, bb) + term(pa * dgt, bb) + term(pa * gt, dbb)
                       + 2 * (e + 4) * U * prod + U * np.abs(logp.reshape(B, L, 16)[:, t])[:, None, :] + 1e-6)
    return bound


def _check_tables(tables, ref_tables, bound):
    err = np.abs(tables - ref_tables)
    assert (err <= bound).all(), (err - bound).max()


SHAPES = [("qwen3-4b-bs1", 256), ("27b-class", 256), ("tiny", 64), ("qwen3-4b-batched", 32)]


@pytest.mark.parametrize("name,e", SHAPES)
def test_ctx_maxsum(name, e):
    w = syn.workload(name)
    Emb, H, Pab, Pg, logp, idx, anchor = _inputs(w, e)
    tok, slot, score, q, tables, _, _ = _run(Emb, H, Pab, Pg, logp, idx, anchor, w.B, w.L, w.V)
    assert q is None
    ref = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, w.B, w.L, walk="maxsum")
    _check_tables(tables, ref["tables"], _table_bound(Emb, H, Pab, Pg, logp, idx, anchor, w.B, w.L))
    firm = ref["margin"] >= 1e-3
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])
    np.testing.assert_array_equal(tok[firm], ref["path_tok"][firm])
    np.testing.assert_allclose(score[firm], ref["path_score"][firm], rtol=1e-5, atol=1e-4)
    idx3 = idx.reshape(w.B, w.L, 16)
    assert (np.take_along_axis(idx3, slot[:, :, None].astype(np.int64), axis=2)[:, :, 0] == tok).all()


@pytest.mark.parametrize("name,e", SHAPES)
def test_ctx_greedy_and_sample(name, e):
    w = syn.workload(name)
    Emb, H, Pab, Pg, logp, idx, anchor = _inputs(w, e, seed_off=1)
    tok, slot, score, _, tables, _, _ = _run(Emb, H, Pab, Pg, logp, idx, anchor, w.B, w.L, w.V, walk="greedy")
    ref = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, w.B, w.L, walk="greedy")
    firm = (ref["margin"] >= 1e-3).all(axis=1)
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])
    np.testing.assert_allclose(score[firm], ref["path_score"][firm], rtol=1e-5, atol=1e-4)
    u = syn.uniforms((w.B, w.L), w.seed, "u_walk")
    tok, slot, score, q, tables, _, _ = _run(Emb, H, Pab, Pg, logp, idx, anchor, w.B, w.L, w.V, walk="sample",
                                             u=u, T=0.8)
    ref = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, w.B, w.L, walk="sample", uniforms=u,
                            temperature=0.8)
    firm = (ref["gap"] >= 1e-4).all(axis=1)
    assert firm.mean() > 0.5
    np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])
    np.testing.assert_allclose(q[firm], ref["q"][firm], rtol=0, atol=1e-5)


def test_ctx_hand_case(golden):
    g = golden("ctx_hand.json")
    V, d, e, L = g["V"], g["d"], g["e"], g["L"]
    Emb = np.zeros((V, d), np.float32)
    for v, c, x in g["Emb_nonzero"]:
        Emb[v, c] = x
    # pad d and e with zero components (the GEMMs take N >= 16; the padding adds nothing)
    dp, ep = 128, 16
    Embp = np.zeros((V, dp), np.float32)
    Embp[:, :d] = Emb
    Pab = np.zeros((2 * ep, dp), np.float32)
    Pab[:e, :d] = np.array(g["Pab"], np.float32)[:e]
    Pab[ep:ep + e, :d] = np.array(g["Pab"], np.float32)[e:]
    Pg = np.zeros((ep, dp), np.float32)
    H = np.ones((L, dp), np.float32)
    logp = np.tile(-np.arange(16, dtype=np.float32), (L, 1))
    idx = np.array([[20 * t + k for k in range(16)] for t in range(L)], np.int32)
    bf = syn.f32_to_bf16_bits
    tok, slot, score, _, tables, _, _ = _run(bf(Embp), bf(H), bf(Pab), bf(Pg), logp, idx,
                                             np.array([g["anchor"]], np.int32), 1, L, V)
    k, v = g["table0_entry"]
    assert (tables[0, 0, :, k] == v).all()
    j, k, v = g["table1_entry"]
    assert tables[0, 1, j, k] == v
    assert slot[0].tolist() == g["path_slot"]
    assert tok[0].tolist() == g["path_tok"]
    assert score[0] == g["path_score"]


def test_ctx_with_verification():
    w = syn.workload("qwen3-4b-batched")
    e = 64
    Emb, H, Pab, Pg, logp, idx, anchor = _inputs(w, e, seed_off=2)
    ref = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, w.B, w.L, walk="maxsum")
    rng = np.random.default_rng(9)
    tgt = np.where(rng.random((w.B, w.L)) < 0.3, (ref["path_tok"] + 1) % w.V, ref["path_tok"])
    target = np.concatenate([tgt, rng.integers(0, w.V, (w.B, 1))], axis=1).astype(np.int32)
    tok, slot, score, _, _, acc, nxt = _run(Emb, H, Pab, Pg, logp, idx, anchor, w.B, w.L, w.V, target=target)
    firm = ref["margin"] >= 1e-3
    racc, rnxt = oracle.verify(ref["path_tok"], target)
    np.testing.assert_array_equal(acc[firm], racc[firm])
    np.testing.assert_array_equal(nxt[firm], rnxt[firm])


@pytest.mark.parametrize("B,L,V,d,e", [(3, 16, 3000, 256, 64), (5, 1, 2000, 128, 32), (40, 12, 5000, 256, 128)])
def test_ctx_edge_shapes(B, L, V, d, e):
    """L = 16 (clusters of 8 CTAs, two tables each), L = 1 (one table, no
    cluster) and a batch large enough to run one CTA per block."""
    w = syn.Workload("ctx-edge", B=B, L=L, P=L + 1, d=d, V=V, r=8, sigma=0.3, seed=B + L)
    Emb, H, Pab, Pg, logp, idx, anchor = _inputs(w, e)
    for walk in ("maxsum", "greedy"):
        tok, slot, score, _, tables, _, _ = _run(Emb, H, Pab, Pg, logp, idx, anchor, B, L, V, walk=walk)
        ref = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, B, L, walk=walk)
        _check_tables(tables, ref["tables"], _table_bound(Emb, H, Pab, Pg, logp, idx, anchor, B, L))
        firm = ref["margin"] >= 1e-3 if walk == "maxsum" else (ref["margin"] >= 1e-3).all(axis=1)
        assert firm.mean() > 0.5
        np.testing.assert_array_equal(slot[firm], ref["path_slot"][firm])


@pytest.mark.parametrize("name,e", [("qwen3-4b-bs1", 256), ("tiny", 64)])
def test_ctx_table_rows(name, e):
    """dflash_ctx_table against the exact products on sampled rows (the first
    and last row of every 128-row tile and random ones), under the GEMM's
    a priori fp32 bound; the gate likewise on every row."""
    import block_draft_selection_b200 as bds
    from block_draft_synth import bf16_bits_to_f32
    w = syn.workload(name)
    Emb, H, Pab, Pg, _, _, _ = _inputs(w, e)
    f = lambda b: bf16_bits_to_f32(b).astype(np.float64)
    tab = bds.dflash_ctx_table(dev_bf16(Emb), dev_bf16(Pab)).cpu().numpy()
    gate = bds.dflash_ctx_gate(dev_bf16(H), dev_bf16(Pg)).cpu().numpy()
    assert tab.shape == (w.V, 2 * e) and gate.shape == (w.M, e)
    rng = np.random.default_rng(5)
    rows = sorted({r for t0 in range(0, w.V, 128) for r in (t0, min(w.V, t0 + 128) - 1)}
                  | set(rng.integers(0, w.V, 64).tolist()))
    x, P = f(Emb[rows]), f(Pab)
    d = x.shape[1]
    exact = x @ P.T
    bound = 4 * d * 2.0 ** -23 * (np.abs(x) @ np.abs(P).T) + 1e-6
    assert (np.abs(tab[rows] - exact) <= bound).all()
    xh, G = f(H), f(Pg)
    assert (np.abs(gate - xh @ G.T) <= 4 * d * 2.0 ** -23 * (np.abs(xh) @ np.abs(G).T) + 1e-6).all()


def test_ctx_bad_index_is_reported():
    """A candidate or anchor index outside [0, V) records DFLASH_ERR_BAD_INDEX
    (it is read as token 0, and the call still returns a path of candidates)."""
    import block_draft_selection_b200 as bds
    w = syn.workload("tiny")
    e = 32
    Emb, H, Pab, Pg, logp, idx, anchor = _inputs(w, e)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tab = bds.dflash_ctx_table(dev_bf16(Emb), dev_bf16(Pab))
    gate = bds.dflash_ctx_gate(dev_bf16(H), dev_bf16(Pg))
    for bad_idx, bad_anchor in ((True, False), (False, True)):
        ix = idx.copy()
        an = anchor.copy()
        if bad_idx:
            ix.reshape(-1)[5] = w.V + 7
        if bad_anchor:
            an[0] = -3
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        tok, slot, *_ = bds.dflash_ctx_walk(t(logp), t(ix), t(an), tab, gate, w.B, w.L, w.V, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == bds.DFLASH_ERR_BAD_INDEX
        s = slot.cpu().numpy()
        assert ((s >= 0) & (s < 16)).all()
