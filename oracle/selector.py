"""Path selector: pair scores over neighbouring candidates and a max-sum walk.

"DFlash 2: Keep Drafting Parallel", section "a lightweight path selector": every
pair of adjacent candidates is scored at once, and the only serial part is one
pass over the precomputed scores.  The pages' scorer is
S_t(a,b) = U_t(b) + <A(a) (.) H(h_t), B(b)>, with trained tables the pages do
not publish; this library fixes a seeded stand-in of the same shape (a unary
term from the drafter plus a low-rank bilinear pair term):

    S_i[j,k] = lp_i(c_ij) + lp_{i+1}(c_{i+1,k}) + e_{c_ij} . M . e_{c_{i+1,k}}

where c_ij is candidate j of position i, lp its log-probability, e a row of the
rank-r table E and M an r x r matrix.  The walk is max-sum (Viterbi) over the
L drafted positions:

    delta_0[j] = 0
    delta_{i+1}[k] = max_j (delta_i[j] + S_i[j,k])      (ties: lowest j)
    final slot = argmax_k delta_{L-1}[k]                  (ties: lowest k)

so a path's score is the sum of its L-1 pair scores.  With L = 1 there are
no pairs: the path is slot 0 with score 0.
"""
import numpy as np

from ._widen import bf16, f32


def pair_scores(topk_logp, topk_idx, E_bits, M_bits, B: int, L: int) -> np.ndarray:
    """S [B, L-1, K, K] float64 from the candidate lists [B*L, K]."""
    lp = f32(topk_logp).reshape(B, L, -1)
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, -1)
    K = lp.shape[2]
    E = bf16(E_bits)
    Msel = bf16(M_bits)
    e = E[idx]                       # [B, L, K, r]
    u = e @ Msel                     # e_c . M, [B, L, K, r]
    S = np.empty((B, max(L - 1, 0), K, K))
    for i in range(L - 1):
        bil = np.einsum("bjr,bkr->bjk", u[:, i], e[:, i + 1])
        S[:, i] = lp[:, i, :, None] + lp[:, i + 1, None, :] + bil
    return S


def viterbi(S: np.ndarray, L: int, K: int = 16):
    """Max-sum walk.  Returns (slots [B, L] int64, score [B] float64)."""
    B = S.shape[0]
    slots = np.zeros((B, L), dtype=np.int64)
    if L == 1:
        return slots, np.zeros(B)
    delta = np.zeros((B, K))
    back = np.zeros((B, L - 1, K), dtype=np.int64)
    for i in range(L - 1):
        cand = delta[:, :, None] + S[:, i]          # [B, j, k]
        back[:, i] = cand.argmax(axis=1)            # first max = lowest j
        delta = cand.max(axis=1)
    last = delta.argmax(axis=1)                     # first max = lowest k
    score = delta[np.arange(B), last]
    slots[:, L - 1] = last
    for i in range(L - 2, -1, -1):
        slots[:, i] = back[np.arange(B), i, slots[:, i + 1]]
    return slots, score


def viterbi_two_best(S: np.ndarray, L: int, K: int = 16):
    """Best and second-best path scores per block (2-best list Viterbi): each
    state keeps its two best distinct partial paths.  Returns (best, second)."""
    B = S.shape[0]
    if L == 1:
        return np.zeros(B), np.zeros(B)     # K single-slot paths, all score 0
    d1 = np.zeros((B, K))
    d2 = np.full((B, K), -np.inf)
    for i in range(L - 1):
        c1 = d1[:, :, None] + S[:, i]               # [B, j, k]
        c2 = d2[:, :, None] + S[:, i]
        allc = np.concatenate([c1, c2], axis=1)     # [B, 2K, k]
        allc.sort(axis=1)
        d1 = allc[:, -1, :]
        d2 = allc[:, -2, :]
    ends = np.concatenate([d1, d2], axis=1)
    ends.sort(axis=1)
    return ends[:, -1], ends[:, -2]


def path_select(topk_logp, topk_idx, E_bits, M_bits, B: int, L: int, K: int = 16):
    """Returns dict with path_tok [B,L], path_slot [B,L], path_score [B],
    margin [B] (best minus second-best path score) and the pair scores."""
    S = pair_scores(topk_logp, topk_idx, E_bits, M_bits, B, L)
    slots, score = viterbi(S, L, K)
    best, second = viterbi_two_best(S, L, K)
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, K)
    tok = np.take_along_axis(idx, slots[:, :, None], axis=2)[:, :, 0]
    return {"path_tok": tok, "path_slot": slots, "path_score": score,
            "margin": best - second, "pair_scores": S}
