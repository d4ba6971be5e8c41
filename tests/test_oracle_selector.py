"""Pins for the oracle's pair scorer and max-sum walk (no GPU).

The exhaustive reference enumerates all 16^L paths (L <= 4) over a pair-score
table computed in exact rational arithmetic straight from the bf16 / fp32 bit
patterns, independent of the oracle's numpy path."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

import oracle
from block_draft_synth import f32_to_bf16_bits, synthetic_topk, rng_for
from exact import exact_pairs

K = 16


def _tables(seed, V, r, scale):
    rng = rng_for(seed, "E")
    E = f32_to_bf16_bits((scale * rng.standard_normal((V, r))).astype(np.float32))
    M = f32_to_bf16_bits((scale * rng.standard_normal((r, r))).astype(np.float32))
    return E, M


_exact_pairs = exact_pairs


def _brute(S, L):
    scored = []
    for path in itertools.product(range(K), repeat=L):
        s = sum((S[i][path[i]][path[i + 1]] for i in range(L - 1)), Fraction(0))
        scored.append((s, path))
    scored.sort(key=lambda t: t[0], reverse=True)
    return scored[0], scored[1]


@pytest.mark.parametrize("L,scale,seed", [(2, 1.0, 0), (3, 0.3, 1), (3, 1.5, 2), (4, 1.0, 3)])
def test_exhaustive_enumeration(L, scale, seed):
    B, V, r = 2, 500, 8
    logp, idx = synthetic_topk(B, L, V, seed)
    E, M = _tables(seed, V, r, scale)
    out = oracle.path_select(logp, idx, E, M, B, L)
    for b in range(B):
        S = _exact_pairs(logp, idx, E, M, b, L)
        np.testing.assert_allclose(out["pair_scores"][b],
                                   [[[float(x) for x in row] for row in Si] for Si in S],
                                   rtol=1e-13, atol=1e-13)
        (s1, p1), (s2, _) = _brute(S, L)
        assert s1 > s2                       # unique optimum in these draws
        assert tuple(out["path_slot"][b]) == p1
        assert out["path_score"][b] == pytest.approx(float(s1), abs=1e-12)
        assert out["margin"][b] == pytest.approx(float(s1 - s2), abs=1e-12)
        assert list(out["path_tok"][b]) == [int(idx[b * L + i, p1[i]]) for i in range(L)]


def test_hand_case(golden):
    g = golden("viterbi_hand.json")
    B, L, V, r = g["B"], g["L"], g["V"], g["r"]
    logp = np.tile(-np.arange(K, dtype=np.float32), (B * L, 1))
    idx = np.array([[100 * i + j for j in range(K)] for i in range(L)], dtype=np.int32)
    E = np.zeros((V, r), dtype=np.float32)
    for v, s, x in g["E_nonzero"]:
        E[v, s] = x
    M = np.zeros((r, r), dtype=np.float32)
    for s, t, x in g["M_nonzero"]:
        M[s, t] = x
    out = oracle.path_select(logp, idx, f32_to_bf16_bits(E), f32_to_bf16_bits(M), B, L)
    assert out["path_slot"][0].tolist() == g["path_slot"]
    assert out["path_tok"][0].tolist() == g["path_tok"]
    assert out["path_score"][0] == g["path_score"]
    assert out["margin"][0] == g["margin"]


def test_zero_pair_term_gives_top1_path():
    """E = 0: path score = lp_0 + 2*sum_{0<i<L-1} lp_i + lp_{L-1}, maximised by
    slot 0 everywhere (the per-position top-1)."""
    B, L, V, r = 5, 7, 1000, 16
    logp, idx = synthetic_topk(B, L, V, 21)
    E = np.zeros((V, r), dtype=np.uint16)
    M = f32_to_bf16_bits(np.ones((r, r), dtype=np.float32))
    out = oracle.path_select(logp, idx, E, M, B, L)
    assert (out["path_slot"] == 0).all()
    lp = logp.astype(np.float64).reshape(B, L, K)
    want = lp[:, 0, 0] + 2 * lp[:, 1:L - 1, 0].sum(axis=1) + lp[:, L - 1, 0]
    np.testing.assert_allclose(out["path_score"], want, rtol=0, atol=1e-12)


def test_single_position():
    logp, idx = synthetic_topk(3, 1, 100, 2)
    E, M = _tables(2, 100, 8, 1.0)
    out = oracle.path_select(logp, idx, E, M, 3, 1)
    assert (out["path_slot"] == 0).all()
    assert (out["path_score"] == 0).all()
    assert (out["path_tok"][:, 0] == idx[:, 0]).all()


def test_transposed_matrix_is_caught():
    """Plant e_b . M . e_a instead of e_a . M . e_b in a copy of the scorer;
    the exact table disagrees (M is not symmetric)."""
    B, L, V, r = 1, 2, 200, 8
    logp, idx = synthetic_topk(B, L, V, 5)
    E, M = _tables(5, V, r, 1.0)
    wrong = oracle.pair_scores(logp, idx, E, M.reshape(r, r).T.copy(), B, L)
    S = _exact_pairs(logp, idx, E, M, 0, L)
    assert np.abs(wrong[0] - np.array([[[float(x) for x in row] for row in Si] for Si in S])).max() > 1e-3
