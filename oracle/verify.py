"""Greedy verification of a drafted block.

"DFlash 2: Keep Drafting Parallel", Table 1 and its caption: the accepted
length counts the verifier's next token.  At temperature 0 the target keeps
the longest prefix of the draft that equals its own argmax tokens, then emits
its own token at the first position that differs (or after the block when all
match).  Table 1's printed lengths (4.27, 6.79) follow from this definition;
the tests pin that.
"""
import numpy as np


def verify(draft, target):
    """draft [B, L], target [B, L+1] (the target's argmax at each drafted
    position plus the bonus position).  Returns (accept_len [B], next_token [B])
    with accept_len = n + 1 where n is the first i with draft[i] != target[i]
    (n = L when every position matches) and next_token = target[n]."""
    draft = np.asarray(draft, dtype=np.int64)
    target = np.asarray(target, dtype=np.int64)
    B, L = draft.shape
    differs = draft != target[:, :L]                  # [B, L]
    n = np.where(differs.any(axis=1), differs.argmax(axis=1), L)   # first difference
    return n + 1, target[np.arange(B), n]
