"""Greedy verification on the GPU against the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn

pytestmark = pytest.mark.gpu


def _run(draft, target):
    import block_draft_selection_b200 as bds
    a, n = bds.dflash_verify(torch.from_numpy(np.ascontiguousarray(draft, np.int32)).cuda(),
                             torch.from_numpy(np.ascontiguousarray(target, np.int32)).cuda())
    return a.cpu().numpy(), n.cpu().numpy()


def test_hand_cases(golden):
    for c in golden("verify_hand.json")["cases"]:
        a, n = _run(np.array([c["draft"]]), np.array([c["target"]]))
        assert (int(a[0]), int(n[0])) == (c["accept_len"], c["next_token"]), c["name"]


@pytest.mark.parametrize("B,L,p", [(1, 7, 0.8), (64, 7, 0.5), (16, 5, 0.9), (256, 16, 0.95),
                                   (1000, 1, 0.5), (333, 32, 0.97), (5, 4, 1.0), (9, 4, 0.0)])
def test_random_bit_exact(B, L, p):
    draft, target = syn.synthetic_verify(B, L, 151936, B * 100 + L, p)
    a, n = _run(draft, target)
    ra, rn = oracle.verify(draft, target)
    np.testing.assert_array_equal(a, ra)
    np.testing.assert_array_equal(n, rn)
