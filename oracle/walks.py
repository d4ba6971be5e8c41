"""Other walks over the pair scores, and rejection-sampling verification.

"DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
the only serial part is the walk over the precomputed scores -- starting from
the last verified token it greedily follows the best successor at each step;
sampling draws from the same scores, and rejection sampling restores the
target's exact distribution ("Inco AI's DFlash 2 lifts LLM decoding output
16-25%": greedy selection, sampling, or rejection sampling that preserves the
target model's exact output distribution).

Readings taken here (the pages give no formulas for these steps):
  * the walk starts at the last verified ("anchor") token a; the anchor has
    no unary term, so the score of a first candidate b is
        S_a[k] = lp_0(c_0k) + e_a . M . e_{c_0k}
    and afterwards S_i[j,k] as in the Viterbi walk (selector.pair_scores);
  * greedy: c_0 = argmax_k S_a[k], c_{i+1} = argmax_k S_i[c_i, k] (ties to
    the lowest slot); the path score is S_a[c_0] + sum_i S_i[c_i, c_{i+1}];
  * sampling at temperature T: the successor of the current token is drawn
    from softmax_k(score_k / T) over the 16 candidates, by inverse CDF in slot
    order with a given uniform u (the smallest k whose cumulative probability
    exceeds u); q[i, k] is that distribution at position i;
  * verification (standard speculative sampling): the draft token x_i is
    kept if r_i * q_i(x_i) <= p_i(x_i) (r_i uniform); at the first rejection n
    the target emits a draw from normalize(max(0, p_n - q_n)), and after L
    acceptances a draw from p_L, each by inverse CDF in vocabulary order with
    a given uniform.
"""
import numpy as np

from ._widen import bf16, f32
from .selector import pair_scores


def anchor_scores(topk_logp, topk_idx, E_bits, M_bits, anchor, B: int, L: int) -> np.ndarray:
    """S_a [B, K]: score of each position-0 candidate after the anchor token."""
    lp = f32(topk_logp).reshape(B, L, -1)
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, -1)
    E = bf16(E_bits)
    Msel = bf16(M_bits)
    ea = E[np.asarray(anchor, dtype=np.int64)]            # [B, r]
    u = ea @ Msel                                          # [B, r]
    e0 = E[idx[:, 0]]                                      # [B, K, r]
    return lp[:, 0, :] + np.einsum("br,bkr->bk", u, e0)


def standin_anchored_tables(topk_logp, topk_idx, E_bits, M_bits, anchor, B: int, L: int) -> np.ndarray:
    """Tables [B, L, K, K] of the walk from the anchor with the stand-in
    scorer: table 0 holds S_a in every row (the anchor is one state), table
    i >= 1 is the pair table S_{i-1} between drafted positions i-1 and i."""
    Sa = anchor_scores(topk_logp, topk_idx, E_bits, M_bits, anchor, B, L)
    S = pair_scores(topk_logp, topk_idx, E_bits, M_bits, B, L)
    K = Sa.shape[1]
    T = np.empty((B, L, K, K))
    T[:, 0] = Sa[:, None, :]
    T[:, 1:] = S
    return T


def greedy_walk_tables(T, topk_idx, B: int, L: int):
    """Greedy walk over anchored tables T [B, L, K, K] (table 0's rows are the
    anchor's): s_0 = argmax_k T_0[0, k], s_{i+1} = argmax_k T_{i+1}[s_i, k],
    ties to the lowest slot.  Returns a dict: path_slot, path_tok [B, L],
    path_score [B] (the sum of the chosen entries) and margin [B, L] (chosen
    minus runner-up at each step)."""
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, -1)
    slots = np.zeros((B, L), dtype=np.int64)
    score = np.zeros(B)
    margin = np.zeros((B, L))

    def second_gap(row, k):
        rest = np.delete(row, k)
        return row[k] - rest.max() if rest.size else np.inf

    for b in range(B):
        cur = 0
        for i in range(L):
            row = T[b, i, cur]
            k = int(np.argmax(row))                        # first max = lowest slot
            score[b] += row[k]
            margin[b, i] = second_gap(row, k)
            slots[b, i] = k
            cur = k
    tok = np.take_along_axis(idx, slots[:, :, None], axis=2)[:, :, 0]
    return {"path_slot": slots, "path_tok": tok, "path_score": score, "margin": margin}


def greedy_walk(topk_logp, topk_idx, E_bits, M_bits, anchor, B: int, L: int):
    """Greedy walk from the anchor with the stand-in scorer; see
    greedy_walk_tables for the returned dict."""
    T = standin_anchored_tables(topk_logp, topk_idx, E_bits, M_bits, anchor, B, L)
    return greedy_walk_tables(T, topk_idx, B, L)


def softmax_t(scores: np.ndarray, T: float) -> np.ndarray:
    z = scores / T
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def inverse_cdf(prob: np.ndarray, u: float) -> int:
    """Smallest k with sum_{j<=k} prob[j] > u (prob need not be normalised:
    u is scaled by the total).  Returns len-1 if rounding leaves none."""
    c = np.cumsum(prob)
    k = int(np.searchsorted(c, u * c[-1], side="right"))
    return min(k, len(prob) - 1)


def sample_walk_tables(T, topk_idx, uniforms, temp: float, B: int, L: int):
    """Sampled walk over anchored tables T [B, L, K, K]: the slot at position
    i is drawn from softmax(T_i[s_{i-1}, :] / temp) (s_{-1} = 0, the anchor)
    by inverse CDF with uniforms[b, i].  Returns a dict: path_slot, path_tok
    [B, L], q [B, L, K] (the distribution each slot was drawn from) and gap
    [B, L], the distance of each uniform to the nearest inner cumulative
    boundary (how close each draw came to changing)."""
    idx = np.asarray(topk_idx, dtype=np.int64).reshape(B, L, -1)
    K = idx.shape[2]
    u = np.asarray(uniforms, dtype=np.float64).reshape(B, L)
    slots = np.zeros((B, L), dtype=np.int64)
    q = np.zeros((B, L, K))
    gap = np.zeros((B, L))
    for b in range(B):
        cur = 0
        for i in range(L):
            pr = softmax_t(T[b, i, cur], temp)
            k = inverse_cdf(pr, u[b, i])
            c = np.cumsum(pr)
            gap[b, i] = np.min(np.abs(c[:-1] - u[b, i])) if K > 1 else 1.0
            slots[b, i] = k
            q[b, i] = pr
            cur = k
    tok = np.take_along_axis(idx, slots[:, :, None], axis=2)[:, :, 0]
    return {"path_slot": slots, "path_tok": tok, "q": q, "gap": gap}


def sample_walk(topk_logp, topk_idx, E_bits, M_bits, anchor, uniforms, T: float, B: int, L: int):
    """Sampled walk from the anchor with the stand-in scorer; see
    sample_walk_tables for the returned dict."""
    tables = standin_anchored_tables(topk_logp, topk_idx, E_bits, M_bits, anchor, B, L)
    return sample_walk_tables(tables, topk_idx, uniforms, T, B, L)


def target_probs(z, T: float) -> np.ndarray:
    """p = softmax(z / T) along the last axis, float64, from fp32 logits."""
    x = np.asarray(z, dtype=np.float32).astype(np.float64) / T
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def verify_rejection(draft, draft_slot, cand_idx, draft_q, target_p, u_accept, u_resample):
    """Speculative-sampling verification.

    draft, draft_slot [B,L]; cand_idx [B*L,K]; draft_q [B,L,K]; target_p
    [B,L+1,V] (each row a distribution); u_accept [B,L]; u_resample [B].
    Returns a dict with accept_len [B] (accepted drafts + 1), next_token [B],
    and two margins that say how close each decision came to flipping:
    accept_margin [B,L] = |u*q - p| / max(p, u*q, tiny) at every tested
    position (inf where not tested) and resample_margin [B] = distance of the
    scaled uniform to the nearest other cumulative boundary, relative to the
    residual's total."""
    draft = np.asarray(draft, dtype=np.int64)
    B, L = draft.shape
    slot = np.asarray(draft_slot, dtype=np.int64)
    cand = np.asarray(cand_idx, dtype=np.int64).reshape(B, L, -1)
    q = np.asarray(draft_q, dtype=np.float64)
    p = np.asarray(target_p, dtype=np.float64)
    ua = np.asarray(u_accept, dtype=np.float64).reshape(B, L)
    ur = np.asarray(u_resample, dtype=np.float64).reshape(B)
    accept = np.empty(B, dtype=np.int64)
    nxt = np.empty(B, dtype=np.int64)
    acc_margin = np.full((B, L), np.inf)
    res_margin = np.empty(B)
    for b in range(B):
        n = L
        for i in range(L):
            x = draft[b, i]
            lhs, rhs = ua[b, i] * q[b, i, slot[b, i]], p[b, i, x]
            acc_margin[b, i] = abs(lhs - rhs) / max(lhs, rhs, 1e-300)
            if not lhs <= rhs:
                n = i
                break
        if n == L:
            res = p[b, L].copy()
        else:
            qv = np.zeros(p.shape[2])
            qv[cand[b, n]] = q[b, n]
            res = np.maximum(0.0, p[b, n] - qv)
        accept[b] = n + 1
        nxt[b] = inverse_cdf(res, ur[b])
        c = np.cumsum(res)
        t = ur[b] * c[-1]
        bounds = c[res > 0][:-1] if (res > 0).sum() > 1 else np.array([np.inf])
        res_margin[b] = np.min(np.abs(bounds - t)) / c[-1]
    return {"accept_len": accept, "next_token": nxt,
            "accept_margin": acc_margin, "resample_margin": res_margin}
