"""Pins for the oracle's LM head + log-softmax + top-16 (no GPU).

The exact reference here is independent of the oracle's numpy path: logits
are computed in exact rational arithmetic from the bf16 bit patterns, the
log-sum-exp in 50-digit decimal arithmetic, and the top-16 by a heap over
exact values."""
import decimal
import heapq
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from block_draft_synth import f32_to_bf16_bits, rng_for


def _bits_to_fraction(b):
    """bf16 bit pattern -> exact Fraction (finite values only)."""
    b = int(b)
    sign = -1 if b & 0x8000 else 1
    exp = (b >> 7) & 0xFF
    man = b & 0x7F
    if exp == 0:
        return sign * Fraction(man, 1 << (126 + 7))
    return sign * Fraction(128 + man, 128) * (Fraction(2) ** (exp - 127))


def _tiny(seed, M=3, V=40, d=8, scale=1.0):
    rng = rng_for(seed, "H")
    H = f32_to_bf16_bits(rng.standard_normal((M, d)).astype(np.float32))
    W = f32_to_bf16_bits((scale * rng.standard_normal((V, d)) / np.sqrt(d)).astype(np.float32))
    return H, W


def _exact(H, W, K):
    M, d = H.shape
    V = W.shape[0]
    Hf = [[_bits_to_fraction(H[m, k]) for k in range(d)] for m in range(M)]
    Wf = [[_bits_to_fraction(W[v, k]) for k in range(d)] for v in range(V)]
    out = []
    ctx = decimal.Context(prec=50)
    for m in range(M):
        z = [sum(Hf[m][k] * Wf[v][k] for k in range(d)) for v in range(V)]
        zd = [ctx.divide(decimal.Decimal(q.numerator), decimal.Decimal(q.denominator)) for q in z]
        lse = ctx.ln(sum((ctx.exp(x) for x in zd), decimal.Decimal(0)))
        top = heapq.nsmallest(K, ((-z[v], v) for v in range(V)))
        out.append((z, lse, [v for _, v in top]))
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_exact_bruteforce(seed):
    H, W = _tiny(seed)
    K = 16
    logp, idx, lse, z = oracle.lmhead_topk(H, W, K, return_logits=True)
    for m, (zq, lse_ex, top_ex) in enumerate(_exact(H, W, K)):
        np.testing.assert_allclose(z[m], [float(q) for q in zq], rtol=0, atol=1e-14)
        assert abs(lse[m] - float(lse_ex)) < 1e-12
        assert idx[m].tolist() == top_ex
        want = [float(decimal.Decimal(zq[v].numerator) / decimal.Decimal(zq[v].denominator) - lse_ex)
                for v in top_ex]
        np.testing.assert_allclose(logp[m], want, rtol=0, atol=1e-12)


def test_ties_resolve_to_lowest_index():
    H, W = _tiny(5, M=2, V=40)
    W = W.copy()
    W[3] = W[17]          # v=3 and v=17 tie exactly
    W[30] = W[17]
    z = oracle.logits(H, W)
    _, idx, _ = oracle.lmhead_topk(H, W, 16)
    for m in range(2):
        order = heapq.nsmallest(40, ((-z[m, v], v) for v in range(40)))
        assert idx[m].tolist() == [v for _, v in order[:16]]
        pos = {v: k for k, v in enumerate(idx[m].tolist())}
        if 3 in pos and 17 in pos:
            assert pos[3] < pos[17]


def test_uniform_logits():
    V, d = 300, 16
    H = f32_to_bf16_bits(np.ones((2, d), dtype=np.float32))
    W = np.zeros((V, d), dtype=np.uint16)          # +0.0 in bf16
    logp, idx, lse = oracle.lmhead_topk(H, W, 16)
    np.testing.assert_allclose(lse, math.log(V), rtol=0, atol=1e-13)
    np.testing.assert_allclose(logp, -math.log(V), rtol=0, atol=1e-13)
    assert idx.tolist() == [list(range(16))] * 2


def test_normalisation_and_order_invariants():
    H, W = _tiny(9, M=4, V=2000, d=64)
    logp, idx, lse, z = oracle.lmhead_topk(H, W, 16, return_logits=True)
    full = z - lse[:, None]
    np.testing.assert_allclose(np.exp(full).sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (logp <= 0).all()
    assert (np.diff(logp, axis=1) <= 0).all()


def test_argmax_tokens_exact():
    H, W = _tiny(4, M=3, V=40)
    got = oracle.argmax_tokens(H, W)
    for m, (zq, _, top) in enumerate(_exact(H, W, 1)):
        assert got[m] == top[0]


def test_transposed_operand_is_caught():
    """A plausible slip -- projecting with W's columns instead of its rows --
    gives a different list than the exact reference (square case so it runs)."""
    H, W = _tiny(6, M=2, V=8, d=8)
    wrong_z = oracle.logits(H, W.T.copy())
    ex = _exact(H, W, 8)
    assert any(np.argsort(-wrong_z[m], kind="stable")[:8].tolist() != ex[m][2] for m in range(2))


def test_margin_comparator():
    rng = np.random.default_rng(0)
    z = rng.standard_normal(500)
    z[10] = 5.0
    z[11] = 5.0 + 5e-4        # near tie with 10
    lse = float(np.log(np.exp(z).sum()))
    exact = np.lexsort((np.arange(500), -z))[:16]
    ok, _ = oracle.topk_margin_ok(z, lse, exact, z[exact] - lse)
    assert ok
    swapped = exact.copy()
    swapped[[0, 1]] = swapped[[1, 0]]
    ok, _ = oracle.topk_margin_ok(z, lse, swapped, z[swapped] - lse)
    assert ok                                    # near tie may swap
    bad = exact.copy()
    bad[[2, 3]] = bad[[3, 2]]
    if abs(z[bad[2]] - z[bad[3]]) >= 1e-3:
        ok, _ = oracle.topk_margin_ok(z, lse, bad, z[bad] - lse)
        assert not ok
    ok, _ = oracle.topk_margin_ok(z, lse, exact, z[exact] - lse + 0.05)
    assert not ok                                # logp tolerance enforced
