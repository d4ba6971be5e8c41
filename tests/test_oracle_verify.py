"""Pins for the oracle's greedy verification (no GPU)."""
import math

import numpy as np

import oracle
from block_draft_synth import synthetic_verify


def test_hand_cases(golden):
    for c in golden("verify_hand.json")["cases"]:
        a, n = oracle.verify(np.array([c["draft"]]), np.array([c["target"]]))
        assert (int(a[0]), int(n[0])) == (c["accept_len"], c["next_token"]), c["name"]


def _closed_form(p):
    # E[accept] = 1 + sum_{k=1..L} prod_{i<k} p_i  (prefix length + the verifier's token)
    return 1.0 + sum(math.prod(p[:k]) for k in range(1, len(p) + 1))


def test_table1_closed_form_matches_printed_lengths(golden):
    t = golden("table1_recall.json")
    for key in ("recall_at_1", "recall_at_16"):
        tau = _closed_form(t[key])
        printed = t["accept_len_printed"][key]
        # the page prints two decimals, truncated
        assert math.floor(tau * 100) / 100 == printed, (key, tau, printed)


def test_table1_statistical(golden):
    """Blocks whose position i matches with probability p_i (Table 1's
    conditional recalls) must have a mean accepted length equal to the closed
    form; this fixes L = 7, the +1 bonus token and the first-mismatch rule."""
    t = golden("table1_recall.json")
    B = 400_000
    for key, seed in (("recall_at_1", 11), ("recall_at_16", 12)):
        p = t[key]
        draft, target = synthetic_verify(B, len(p), 151936, seed, p)
        acc, nxt = oracle.verify(draft, target)
        tau = _closed_form(p)
        se = acc.std() / math.sqrt(B)
        assert abs(acc.mean() - tau) < 5 * se, (key, acc.mean(), tau, se)
        assert acc.min() >= 1 and acc.max() <= len(p) + 1


def test_invariants_random():
    draft, target = synthetic_verify(5000, 9, 1000, 3, 0.7)
    acc, nxt = oracle.verify(draft, target)
    L = draft.shape[1]
    for b in range(0, 5000, 97):
        n = acc[b] - 1
        assert np.array_equal(draft[b, :n], target[b, :n])
        assert n == L or draft[b, n] != target[b, n]
        assert nxt[b] == target[b, n]
