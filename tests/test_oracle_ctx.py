"""Pins for the oracle's context-gated scorer (no GPU): a hand-worked case,
exact rational tables with the gate fixed at 1/2 (zero gate projection), at 1
(saturated gate) and switching between 1 and 0 from one position to the next
(which hidden state gates which table), brute force over every anchored path,
the zero projection case and planted slips (the two projections swapped; the
gate taken from the neighbouring position)."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

import oracle
from block_draft_synth import f32_to_bf16_bits, synthetic_topk, rng_for
from exact import bf

K = 16


def _hand(g):
    V, d = g["V"], g["d"]
    Emb = np.zeros((V, d), np.float32)
    for v, c, x in g["Emb_nonzero"]:
        Emb[v, c] = x
    Pab = np.array(g["Pab"], np.float32)
    Pg = np.zeros((g["e"], d), np.float32)
    L = g["L"]
    logp = np.tile(-np.arange(K, dtype=np.float32), (L, 1))
    idx = np.array([[20 * t + k for k in range(K)] for t in range(L)], np.int32)
    H = f32_to_bf16_bits(np.ones((L, d), np.float32))
    return logp, idx, f32_to_bf16_bits(Emb), H, f32_to_bf16_bits(Pab), f32_to_bf16_bits(Pg)


def test_hand_case(golden):
    g = golden("ctx_hand.json")
    logp, idx, Emb, H, Pab, Pg = _hand(g)
    B, L = g["B"], g["L"]
    anchor = [g["anchor"]]
    T = oracle.ctx_tables(logp, idx, Emb, H, Pab, Pg, anchor, B, L)
    k, v = g["table0_entry"]
    assert (T[0, 0, :, k] == v).all()                       # every row: the anchor
    j, k, v = g["table1_entry"]
    assert T[0, 1, j, k] == v
    gr = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, B, L, walk="greedy")
    ms = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, B, L, walk="maxsum")
    for out in (gr, ms):
        assert out["path_slot"][0].tolist() == g["path_slot"]
        assert out["path_tok"][0].tolist() == g["path_tok"]
        assert out["path_score"][0] == g["path_score"]
    assert ms["margin"][0] == g["margin"]


def _random(seed, B, L, V, d, e, gate_scale):
    rng = rng_for(seed, "gate")
    logp, idx = synthetic_topk(B, L, V, seed)
    bfr = lambda shape, s: f32_to_bf16_bits((s * rng.standard_normal(shape)).astype(np.float32))
    Emb = bfr((V, d), 1.0)
    H = bfr((B * L, d), 1.0)
    Pab = bfr((2 * e, d), 0.5)
    Pg = bfr((e, d), gate_scale) if gate_scale else np.zeros((e, d), np.uint16)
    anchor = rng.integers(0, V, size=B)
    return logp, idx, Emb, H, Pab, Pg, anchor


def _exact_tables(logp, idx, Emb, Pab, anchor, b, L, e, gate):
    """Tables from Fractions of the bit patterns, with a fixed gate value
    (one Fraction for every table, or a list: table t gated by gate[t])."""
    gates = list(gate) if isinstance(gate, (list, tuple)) else [gate] * L
    d = Emb.shape[1]
    proj = lambda tok, rows: [sum(bf(Emb[tok, c]) * bf(Pab[q, c]) for c in range(d)) for q in rows]
    A = lambda tok: proj(tok, range(e))
    Bp = lambda tok: proj(tok, range(e, 2 * e))
    lp = lambda t, k: Fraction(float(logp[b * L + t, k]))
    T = []
    for t in range(L):
        preds = [A(int(anchor[b]))] * K if t == 0 else [A(int(idx[b * L + t - 1, j])) for j in range(K)]
        succ = [Bp(int(idx[b * L + t, k])) for k in range(K)]
        T.append([[lp(t, k) + sum(preds[j][q] * gates[t] * succ[k][q] for q in range(e)) for k in range(K)]
                  for j in range(K)])
    return T


@pytest.mark.parametrize("L,seed", [(1, 0), (2, 1), (3, 2)])
def test_exact_tables_and_brute_force(L, seed):
    """Gate 1/2 (zero gate projection): tables equal the exact rational ones;
    the max-sum walk equals brute force over all 16^L anchored paths."""
    B, V, d, e = 2, 120, 8, 4
    logp, idx, Emb, H, Pab, Pg, anchor = _random(seed, B, L, V, d, e, 0.0)
    out = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, B, L, walk="maxsum")
    for b in range(B):
        T = _exact_tables(logp, idx, Emb, Pab, anchor, b, L, e, Fraction(1, 2))
        np.testing.assert_allclose(out["tables"][b], [[[float(x) for x in r] for r in Tt] for Tt in T],
                                   rtol=1e-13, atol=1e-12)
        scored = []
        for path in itertools.product(range(K), repeat=L):
            s = T[0][0][path[0]] + sum((T[t][path[t - 1]][path[t]] for t in range(1, L)), Fraction(0))
            scored.append((s, path))
        scored.sort(key=lambda z: z[0], reverse=True)
        (s1, p1), (s2, _) = scored[0], scored[1]
        assert tuple(out["path_slot"][b]) == p1
        assert out["path_score"][b] == pytest.approx(float(s1), abs=1e-12)
        assert out["margin"][b] == pytest.approx(float(s1 - s2), abs=1e-12)


def test_saturated_gate_is_plain_bilinear():
    """A gate projection driven far positive makes H(h) = 1 exactly in fp64:
    the tables are lp + <A, B>."""
    B, L, V, d, e = 1, 2, 100, 8, 4
    logp, idx, Emb, H, Pab, _, anchor = _random(5, B, L, V, d, e, 0.0)
    H1 = f32_to_bf16_bits(np.ones((B * L, d), np.float32))
    Pg = f32_to_bf16_bits(np.full((e, d), 64.0, np.float32))   # Pg.h = 512: sigmoid = 1 - 4e-223
    T = oracle.ctx_tables(logp, idx, Emb, H1, Pab, Pg, anchor, B, L)
    ex = _exact_tables(logp, idx, Emb, Pab, anchor, 0, L, e, Fraction(1))
    np.testing.assert_allclose(T[0], [[[float(x) for x in r] for r in Tt] for Tt in ex], rtol=1e-13, atol=1e-12)


def test_zero_projection_is_top1():
    B, L, V, d, e = 3, 5, 200, 8, 4
    logp, idx, Emb, H, _, Pg, anchor = _random(6, B, L, V, d, e, 1.0)
    Pab = np.zeros((2 * e, d), np.uint16)
    for walk in ("maxsum", "greedy"):
        out = oracle.ctx_select(logp, idx, Emb, H, Pab, Pg, anchor, B, L, walk=walk)
        assert (out["path_slot"] == 0).all()
    lp = logp.astype(np.float64).reshape(B, L, K)
    T = oracle.ctx_tables(logp, idx, Emb, H, Pab, Pg, anchor, B, L)
    np.testing.assert_array_equal(T, np.broadcast_to(lp[:, :, None, :], T.shape))


def test_planted_projection_swap_is_caught():
    """Scoring with Pb on the predecessor and Pa on the candidate (a copy,
    on the CPU) gives different tables from the exact ones."""
    B, L, V, d, e = 1, 2, 100, 8, 4
    logp, idx, Emb, H, Pab, Pg, anchor = _random(7, B, L, V, d, e, 0.0)
    swapped = np.concatenate([Pab[e:], Pab[:e]])
    wrong = oracle.ctx_tables(logp, idx, Emb, H, swapped, Pg, anchor, B, L)
    ex = _exact_tables(logp, idx, Emb, Pab, anchor, 0, L, e, Fraction(1, 2))
    assert np.abs(wrong[0] - np.array([[[float(x) for x in r] for r in Tt] for Tt in ex])).max() > 1e-3


def test_gate_is_a_sigmoid():
    assert oracle.ctx_scorer.sigmoid(0.0) == 0.5
    x = np.array([-3.0, 0.5, 4.0])
    np.testing.assert_allclose(oracle.ctx_scorer.sigmoid(x) + oracle.ctx_scorer.sigmoid(-x), 1.0, rtol=0,
                               atol=1e-15)
    assert oracle.ctx_scorer.sigmoid(np.log(3.0)) == pytest.approx(0.75, rel=1e-15)


def _alternating_gate_case(L, seed):
    """Hidden states +1 at even positions and -1 at odd ones with Pg = 64
    everywhere (d = 8): Pg.h_t = +-512, so the gate is 1 at even t and
    sigmoid(-512) ~ 4e-223 (0 to far below any tolerance) at odd t."""
    B, V, d, e = 2, 150, 8, 4
    logp, idx, Emb, _, Pab, _, anchor = _random(seed, B, L, V, d, e, 0.0)
    sign = np.where(np.arange(B * L) % L % 2 == 0, 1.0, -1.0).astype(np.float32)
    H = f32_to_bf16_bits(sign[:, None] * np.ones((B * L, d), np.float32))
    Pg = f32_to_bf16_bits(np.full((e, d), 64.0, np.float32))
    gates = [Fraction(1) if t % 2 == 0 else Fraction(0) for t in range(L)]
    return B, e, logp, idx, Emb, H, Pab, Pg, anchor, gates


def _as_float(T):
    return np.array([[[float(x) for x in r] for r in Tt] for Tt in T])


@pytest.mark.parametrize("L,seed", [(3, 11), (4, 12)])
def test_gate_follows_own_position(L, seed):
    """Table t is gated by the hidden state at position t: with gates that
    alternate 1, 0, 1, ... the tables equal the exact rational ones whose
    table t carries the gate of position t (S_t(a, b) = U_t(b) +
    <A(a) (.) H(h_t), B(b)>, "DFlash 2: Keep Drafting Parallel", section "a
    lightweight path selector")."""
    B, e, logp, idx, Emb, H, Pab, Pg, anchor, gates = _alternating_gate_case(L, seed)
    T = oracle.ctx_tables(logp, idx, Emb, H, Pab, Pg, anchor, B, L)
    for b in range(B):
        ex = _as_float(_exact_tables(logp, idx, Emb, Pab, anchor, b, L, e, gates))
        np.testing.assert_allclose(T[b], ex, rtol=1e-13, atol=1e-12)
        # the gated-off tables are the unary term alone
        for t in range(1, L, 2):
            np.testing.assert_allclose(T[b, t], np.broadcast_to(logp[b * L + t].astype(np.float64), (K, K)),
                                       rtol=0, atol=1e-12)


@pytest.mark.parametrize("shift", [1, -1])
def test_planted_gate_position_slip_is_caught(shift):
    """Gating table t with h_{t-1} (shift 1) or h_{t+1} (shift -1): the same
    oracle fed hidden states moved by one position (a copy, on the CPU) gives
    tables that miss the exact ones by far more than any tolerance."""
    L = 4
    B, e, logp, idx, Emb, H, Pab, Pg, anchor, gates = _alternating_gate_case(L, 13)
    Hs = np.roll(H.reshape(B, L, -1), shift, axis=1).reshape(B * L, -1)
    wrong = oracle.ctx_tables(logp, idx, Emb, Hs, Pab, Pg, anchor, B, L)
    for b in range(B):
        ex = _as_float(_exact_tables(logp, idx, Emb, Pab, anchor, b, L, e, gates))
        assert np.abs(wrong[b] - ex).max() > 1e-3
