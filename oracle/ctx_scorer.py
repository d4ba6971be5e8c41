"""The pages' context-gated pair scorer, float64 (test infrastructure).

"DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
for the previous token a and a candidate b at position t,

    S_t(a, b) = U_t(b) + < A(a) (.) H(h_t), B(b) >

U_t(b) is the drafter's own logit for b; A and B give every token a compact
256-dimensional embedding; H(h_t), computed from the drafter's hidden state at
position t, gates which components of the match count.  Table 2 prices the
selector at 2.0M parameters.

Readings taken here (the pages give no formulas for A, B or H):
  * A(a) = Pa . emb(a) and B(b) = Pb . emb(b): two e x d projections of the
    token embedding emb = Emb[token] (Emb [V, d]), stored together as
    Pab [2e, d] (rows 0..e-1 = Pa, rows e..2e-1 = Pb);
  * H(h_t) = sigmoid(Pg . h_t) with Pg [e, d]: a gate in (0, 1) per
    component; 3 e d = 1.97M parameters at e = 256, d = 2560 (the 2.0M);
  * U_t(b) enters as the drafter's log-probability (logit minus the row's
    log-sum-exp, a per-position constant: every walk picks the same path);
  * the walk starts at the last verified token (the anchor); position 0's
    predecessor is the anchor, position t's is the token chosen at t-1.

The tables returned are anchored tables [B, L, K, K]: table t holds
S_t(a_j, c_tk) with row j = the predecessor's slot (all rows equal for
t = 0: the anchor is one state) and column k = the candidate's slot.
"""
import numpy as np

from ._widen import bf16, f32
from .selector import viterbi
from .walks import greedy_walk_tables, sample_walk_tables


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def ctx_tables(topk_logp, topk_idx, Emb_bits, H_bits, Pab_bits, Pg_bits, anchor, B: int, L: int) -> np.ndarray:
    """Anchored tables [B, L, K, K] of the context-gated scorer."""
    lp = f32(topk_logp).reshape(B, L, -1)
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, -1)
    K = lp.shape[2]
    Emb_bits = np.asarray(Emb_bits)
    H = bf16(H_bits).reshape(B, L, -1)
    Pab = bf16(Pab_bits)
    e = Pab.shape[0] // 2
    Pa, Pb = Pab[:e], Pab[e:]
    Pg = bf16(Pg_bits)
    gate = sigmoid(H @ Pg.T)                               # [B, L, e]
    cand = bf16(Emb_bits[idx])                             # [B, L, K, d]
    A_c = cand @ Pa.T                                      # [B, L, K, e]
    B_c = cand @ Pb.T                                      # [B, L, K, e]
    A_anchor = bf16(Emb_bits[np.asarray(anchor, dtype=np.int64)]) @ Pa.T   # [B, e]
    T = np.empty((B, L, K, K))
    for t in range(L):
        pred = A_anchor[:, None, :].repeat(K, axis=1) if t == 0 else A_c[:, t - 1]   # [B, K, e]
        w = pred * gate[:, t][:, None, :]
        T[:, t] = lp[:, t][:, None, :] + np.einsum("bjq,bkq->bjk", w, B_c[:, t])
    return T


def maxsum_walk_tables(T, topk_idx, B: int, L: int):
    """Max-sum walk from the anchor over anchored tables: the Viterbi walk
    over L+1 positions whose first is the anchor.  Returns a dict: path_slot,
    path_tok [B, L], path_score [B] and margin [B] (best minus second-best
    path score)."""
    K = T.shape[2]
    slots, score = viterbi(T, L + 1, K)
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, K)
    s = slots[:, 1:]
    tok = np.take_along_axis(idx, s[:, :, None], axis=2)[:, :, 0]
    # the anchor's 16 rows are one state, so the margin is taken over paths
    # of the drafted positions only
    return {"path_slot": s, "path_tok": tok, "path_score": score, "margin": _distinct_margin(T, L, K)}


def _distinct_margin(T, L: int, K: int):
    """Best minus second-best path score over paths of the drafted positions
    (the anchor's copies collapsed to row 0): a 2-best Viterbi whose start is
    the single anchor state."""
    B = T.shape[0]
    d1 = T[:, 0, 0, :].copy()                      # one start state
    d2 = np.full((B, K), -np.inf)
    for t in range(1, L):
        c1 = d1[:, :, None] + T[:, t]
        c2 = d2[:, :, None] + T[:, t]
        allc = np.concatenate([c1, c2], axis=1)
        allc.sort(axis=1)
        d1, d2 = allc[:, -1, :], allc[:, -2, :]
    ends = np.concatenate([d1, d2], axis=1)
    ends.sort(axis=1)
    return ends[:, -1] - ends[:, -2]


def ctx_select(topk_logp, topk_idx, Emb_bits, H_bits, Pab_bits, Pg_bits, anchor, B: int, L: int,
               walk: str = "maxsum", uniforms=None, temperature: float = 1.0):
    """Tables of the context-gated scorer and one walk over them
    ("maxsum", "greedy" or "sample").  Returns the walk's dict plus "tables"."""
    T = ctx_tables(topk_logp, topk_idx, Emb_bits, H_bits, Pab_bits, Pg_bits, anchor, B, L)
    if walk == "maxsum":
        out = maxsum_walk_tables(T, topk_idx, B, L)
    elif walk == "greedy":
        out = greedy_walk_tables(T, topk_idx, B, L)
    elif walk == "sample":
        out = sample_walk_tables(T, topk_idx, uniforms, temperature, B, L)
    else:
        raise ValueError(walk)
    out["tables"] = T
    return out
