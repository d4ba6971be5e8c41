"""Pins for the oracle's greedy and sampling walks and its rejection-sampling
verification (no GPU).

Independent checks: a hand-worked case, exact rational scores, limits with a
closed form, and distributions integrated over grids of uniforms compared with
what the mathematics fixes (the conditional softmaxes of the walk; the
target's own distribution for rejection sampling)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from block_draft_synth import f32_to_bf16_bits, synthetic_topk, rng_for
from exact import exact_pairs, exact_anchor

K = 16


def _tables(seed, V, r, scale):
    rng = rng_for(seed, "E")
    E = f32_to_bf16_bits((scale * rng.standard_normal((V, r))).astype(np.float32))
    M = f32_to_bf16_bits((scale * rng.standard_normal((r, r))).astype(np.float32))
    return E, M


def _hand_tables(g):
    E = np.zeros((g["V"], g["r"]), dtype=np.float32)
    for v, s, x in g["E_nonzero"]:
        E[v, s] = x
    M = np.zeros((g["r"], g["r"]), dtype=np.float32)
    for s, t, x in g["M_nonzero"]:
        M[s, t] = x
    return f32_to_bf16_bits(E), f32_to_bf16_bits(M)


def test_greedy_hand_case(golden):
    g = golden("walks_hand.json")["greedy"]
    B, L = g["B"], g["L"]
    logp = np.tile(-np.arange(K, dtype=np.float32), (B * L, 1))
    idx = np.array([[100 * i + j for j in range(K)] for i in range(L)], dtype=np.int32)
    E, M = _hand_tables(g)
    out = oracle.greedy_walk(logp, idx, E, M, [g["anchor"]], B, L)
    assert out["path_slot"][0].tolist() == g["path_slot"]
    assert out["path_tok"][0].tolist() == g["path_tok"]
    assert out["path_score"][0] == g["path_score"]
    # the anchored max-sum path (1, 10, 0) scores 28: greedy is myopic
    Sa = oracle.anchor_scores(logp, idx, E, M, [g["anchor"]], B, L)
    S = oracle.pair_scores(logp, idx, E, M, B, L)
    assert Sa[0, 1] + S[0, 0, 1, 10] + S[0, 1, 10, 0] == 28.0


@pytest.mark.parametrize("L,scale,seed", [(1, 1.0, 0), (2, 1.0, 1), (4, 0.5, 2), (5, 1.5, 3)])
def test_greedy_exact(L, scale, seed):
    """Greedy steps taken on exact rational scores."""
    B, V, r = 2, 300, 8
    logp, idx = synthetic_topk(B, L, V, seed)
    E, M = _tables(seed, V, r, scale)
    anchor = np.array([7, 123])
    out = oracle.greedy_walk(logp, idx, E, M, anchor, B, L)
    for b in range(B):
        Sa = exact_anchor(logp, idx, E, M, anchor[b], b, L)
        S = exact_pairs(logp, idx, E, M, b, L)
        k = max(range(K), key=lambda j: (Sa[j], -j))
        slots, score = [k], Sa[k]
        for i in range(L - 1):
            nk = max(range(K), key=lambda j: (S[i][k][j], -j))
            score += S[i][k][nk]
            k = nk
            slots.append(k)
        assert out["path_slot"][b].tolist() == slots
        assert out["path_score"][b] == pytest.approx(float(score), abs=1e-12)
        assert out["path_tok"][b].tolist() == [int(idx[b * L + i, s]) for i, s in enumerate(slots)]


def test_greedy_zero_pair_term_is_top1():
    B, L, V, r = 3, 6, 500, 8
    logp, idx = synthetic_topk(B, L, V, 9)
    E = np.zeros((V, r), dtype=np.uint16)
    M = f32_to_bf16_bits(np.ones((r, r), dtype=np.float32))
    out = oracle.greedy_walk(logp, idx, E, M, [0, 1, 2], B, L)
    assert (out["path_slot"] == 0).all()
    lp = logp.astype(np.float64).reshape(B, L, K)
    # S_a[0] = lp_0(0); each pair (0,0) adds lp_i(0) + lp_{i+1}(0)
    want = lp[:, 0, 0] + lp[:, :-1, 0].sum(axis=1) + lp[:, 1:, 0].sum(axis=1)
    np.testing.assert_allclose(out["path_score"], want, rtol=0, atol=1e-12)


def test_inverse_cdf_hand(golden):
    g = golden("walks_hand.json")["inverse_cdf"]
    for u, k in g["cases"]:
        assert oracle.inverse_cdf(np.array(g["prob"]), u) == k


def test_sample_walk_cold_limit_is_greedy():
    B, L, V, r = 4, 5, 400, 8
    logp, idx = synthetic_topk(B, L, V, 11)
    E, M = _tables(11, V, r, 1.0)
    anchor = np.arange(B) * 17
    u = rng_for(11, "gate").uniform(0.0, 1.0 - 1e-6, size=(B, L))
    gr = oracle.greedy_walk(logp, idx, E, M, anchor, B, L)
    assert gr["margin"].min() > 1e-2          # no near-ties in this draw
    sw = oracle.sample_walk(logp, idx, E, M, anchor, u, 1e-4, B, L)
    assert (sw["path_slot"] == gr["path_slot"]).all()


def test_sample_walk_zero_pair_term_closed_form():
    """E = 0, T = 1: every step draws from the drafter's top-16 probabilities
    renormalised, exp(lp) / sum exp(lp), whatever the previous token."""
    B, L, V, r = 2, 4, 300, 8
    logp, idx = synthetic_topk(B, L, V, 13)
    E = np.zeros((V, r), dtype=np.uint16)
    M = f32_to_bf16_bits(np.ones((r, r), dtype=np.float32))
    u = rng_for(13, "gate").uniform(size=(B, L))
    sw = oracle.sample_walk(logp, idx, E, M, [5, 6], u, 1.0, B, L)
    p = np.exp(logp.astype(np.float64)).reshape(B, L, K)
    p /= p.sum(axis=2, keepdims=True)
    np.testing.assert_allclose(sw["q"], p, rtol=1e-12, atol=0)
    for b in range(B):
        for i in range(L):
            c = np.cumsum(p[b, i])
            assert sw["path_slot"][b, i] == int(np.argmax(c > u[b, i]))


def test_sample_walk_distribution():
    """Integrate the walk over a midpoint grid of (u_0, u_1) and compare the
    frequency of every 2-step path with exp(S_a/T)-softmax times the exact
    conditional softmax of the next step."""
    B, L, V, r, T = 1, 2, 200, 8, 0.7
    logp, idx = synthetic_topk(B, L, V, 17, spread=0.3)
    E, M = _tables(17, V, r, 0.8)
    anchor = [42]
    Sa = [float(x) for x in exact_anchor(logp, idx, E, M, anchor[0], 0, L)]
    S0 = [[float(x) for x in row] for row in exact_pairs(logp, idx, E, M, 0, L)[0]]

    def sm(v):
        v = np.array(v) / T
        e = np.exp(v - v.max())
        return e / e.sum()

    want = sm(Sa)[:, None] * np.array([sm(S0[j]) for j in range(K)])
    n = 400
    g = (np.arange(n) + 0.5) / n
    u = np.stack(np.meshgrid(g, g, indexing="ij"), axis=-1).reshape(-1, 2)
    sw = oracle.sample_walk(np.tile(logp, (n * n, 1)), np.tile(idx, (n * n, 1)), E, M,
                            np.full(n * n, anchor[0]), u, T, n * n, L)
    freq = np.zeros((K, K))
    np.add.at(freq, (sw["path_slot"][:, 0], sw["path_slot"][:, 1]), 1.0 / (n * n))
    # each grid dimension resolves probabilities to 1/n
    assert np.abs(freq - want).max() < 2.0 / n


def test_rejection_hand_cases(golden):
    g = golden("walks_hand.json")["rejection"]
    p = np.array(g["p"])[None]
    q = np.array(g["q"])[None, None]
    cand = np.array([g["cand"]])
    for ua, ur, acc, nxt in g["cases"]:
        out = oracle.verify_rejection([[g["draft"]]], [[g["slot"]]], cand, q, p, [[ua]], [ur])
        assert out["accept_len"][0] == acc
        assert out["next_token"][0] == nxt


def _random_case(seed, V, Kc, peaked):
    rng = rng_for(seed, "verify")
    p = rng.dirichlet(np.full(V, 0.5), size=2)             # p_0, p_1
    cand = rng.choice(V, size=Kc, replace=False)
    q = rng.dirichlet(np.full(Kc, 0.3 if peaked else 2.0))
    return p, cand, q


@pytest.mark.parametrize("seed,peaked", [(0, True), (1, False), (2, True)])
def test_rejection_preserves_target_distribution(seed, peaked):
    """Speculative sampling's guarantee: the first emitted token (the draft
    if accepted, else the resampled token) has distribution p_0 exactly.
    Integrated over a midpoint grid of u_accept for each draft slot and a
    grid of u_resample; the grids resolve probabilities to 1/n."""
    V, Kc, n = 9, 4, 4000
    p, cand, q = _random_case(seed, V, Kc, peaked)
    g = (np.arange(n) + 0.5) / n
    first = np.zeros(V)
    for s in range(Kc):
        out = oracle.verify_rejection(np.full((n, 1), cand[s]), np.full((n, 1), s),
                                      np.tile(cand, (n, 1)), np.tile(q, (n, 1, 1)),
                                      np.tile(p, (n, 1, 1)), g[:, None], np.full(n, 0.5))
        acc = out["accept_len"] == 2
        first[cand[s]] += q[s] * acc.mean()
        # rejected blocks: the resampled token's distribution over u_resample
        if (~acc).any():
            rej = oracle.verify_rejection(np.full((n, 1), cand[s]), np.full((n, 1), s),
                                          np.tile(cand, (n, 1)), np.tile(q, (n, 1, 1)),
                                          np.tile(p, (n, 1, 1)), np.ones((n, 1)), g)
            assert (rej["accept_len"] == 1).all()
            np.add.at(first, rej["next_token"], q[s] * (1.0 - acc.mean()) / n)
    np.testing.assert_allclose(first, p[0], atol=3.0 / n)


def test_rejection_always_accepts_when_target_equals_draft():
    V, Kc, L = 7, 3, 3
    rng = rng_for(3, "verify")
    cand = np.stack([rng.choice(V, size=Kc, replace=False) for _ in range(L)])
    q = rng.dirichlet(np.ones(Kc), size=L)
    p = np.zeros((L + 1, V))
    for i in range(L):
        p[i, cand[i]] = q[i]
    p[L] = rng.dirichlet(np.ones(V))
    slot = np.array([0, 2, 1])
    draft = cand[np.arange(L), slot]
    out = oracle.verify_rejection(draft[None], slot[None], cand, q[None], p[None], [[0.999999] * L], [0.3])
    assert out["accept_len"][0] == L + 1
    assert out["next_token"][0] == oracle.inverse_cdf(p[L], 0.3)


def test_rejection_never_resamples_the_rejected_token():
    """A rejection at n implies p_n(x) < q_n(x), so the residual is zero at x."""
    V, Kc = 12, 4
    for seed in range(20):
        p, cand, q = _random_case(seed, V, Kc, True)
        for s in range(Kc):
            for ur in (0.01, 0.5, 0.99):
                out = oracle.verify_rejection([[cand[s]]], [[s]], cand[None], q[None, None], p[None],
                                              [[1.0]], [ur])
                if out["accept_len"][0] == 1:
                    assert out["next_token"][0] != cand[s]
                    assert p[0, out["next_token"][0]] > 0


def test_planted_residual_sign_error_is_caught():
    """A residual of max(0, q - p) instead of max(0, p - q) breaks the
    distribution theorem (mistake planted in a copy, on the CPU)."""
    V, Kc, n = 9, 4, 2000
    p, cand, q = _random_case(0, V, Kc, True)
    g = (np.arange(n) + 0.5) / n

    def wrong_next(s, ur):
        qv = np.zeros(V)
        qv[cand] = q
        return oracle.inverse_cdf(np.maximum(0.0, qv - p[0]), ur)

    first = np.zeros(V)
    for s in range(Kc):
        acc = (g * q[s] <= p[0, cand[s]]).mean()
        first[cand[s]] += q[s] * acc
        for ur in g:
            first[wrong_next(s, ur)] += q[s] * (1 - acc) / n
    assert np.abs(first - p[0]).max() > 10.0 / n


def test_target_probs_closed_forms():
    z = np.log(np.array([[1.0, 2.0, 3.0], [5.0, 5.0, 5.0]], dtype=np.float32))
    p = oracle.target_probs(z, 1.0)
    np.testing.assert_allclose(p[0], [1 / 6, 2 / 6, 3 / 6], rtol=1e-6)
    np.testing.assert_allclose(p[1], [1 / 3] * 3, rtol=1e-15)
    # temperature 2 on log-weights (1, 4, 9) gives weights (1, 2, 3)
    z2 = np.log(np.array([[1.0, 4.0, 9.0]], dtype=np.float32))
    np.testing.assert_allclose(oracle.target_probs(z2, 2.0)[0], [1 / 6, 2 / 6, 3 / 6], rtol=1e-6)
