"""LM-head projection, log-softmax and top-16 candidates, float64.

"DFlash 2: Keep Drafting Parallel", section "the right token is already in the
candidates" and Table 1: the drafter keeps each drafted position's 16 best
candidates; section "a lightweight path selector": those candidates are scored
without another backbone or LM-head pass.  The projection is the drafter's LM
head over the full vocabulary (no bias, temperature 1), normalised by
log-softmax so the kept scores are log-probabilities.

Ordering of the candidate list: value descending, then vocabulary index
ascending (so ties resolve to the lowest index).
"""
import numpy as np

from ._widen import bf16

CHUNK_ROWS = 8192


def logits(H_bits, W_bits, chunk_rows: int = CHUNK_ROWS) -> np.ndarray:
    """z[m, v] = sum_k H[m,k] * W[v,k] in float64 (W widened in row chunks).
    H [M,d], W [V,d] bf16 bits -> z [M,V] float64."""
    H = bf16(H_bits)
    W_bits = np.asarray(W_bits)
    V = W_bits.shape[0]
    z = np.empty((H.shape[0], V))
    for v0 in range(0, V, chunk_rows):
        v1 = min(V, v0 + chunk_rows)
        z[:, v0:v1] = H @ bf16(W_bits[v0:v1]).T
    return z


def log_sum_exp(z: np.ndarray) -> np.ndarray:
    """lse[m] = log sum_v exp(z[m,v]), shifted by the row maximum."""
    zmax = z.max(axis=1)
    return zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))


def top_k_exact(z: np.ndarray, K: int):
    """K largest entries per row by a full stable sort on (-value, index)."""
    M, V = z.shape
    idx = np.empty((M, K), dtype=np.int64)
    for m in range(M):
        order = np.lexsort((np.arange(V), -z[m]))
        idx[m] = order[:K]
    val = np.take_along_axis(z, idx, axis=1)
    return val, idx


def lmhead_topk(H_bits, W_bits, K: int = 16, return_logits: bool = False):
    """Returns (topk_logp [M,K], topk_idx [M,K] int64, lse [M]) and, when
    asked, the full logits z [M,V] (used by the margin-aware comparison)."""
    z = logits(H_bits, W_bits)
    lse = log_sum_exp(z)
    val, idx = top_k_exact(z, K)
    logp = val - lse[:, None]
    if return_logits:
        return logp, idx, lse, z
    return logp, idx, lse


def argmax_tokens(H_bits, W_bits) -> np.ndarray:
    """argmax_v z[m, v], ties to the lowest index: the token a model whose
    final hidden state is H[m] would emit greedily through head W."""
    z = logits(H_bits, W_bits)
    return z.argmax(axis=1)


def topk_margin_ok(z_row: np.ndarray, lse: float, got_idx, got_logp, K: int = 16,
                   margin: float = 1e-3, logp_tol: float = 2e-2):
    """Compare one row's candidate list from another implementation with the
    exact one.  A slot may hold a different index than the exact list only if
    the two indices' exact logits differ by less than ``margin`` (a near-tie
    swap, inside the list or across the 16/17 boundary); every reported
    log-prob must be within ``logp_tol`` of the exact log-prob of the index it
    reports.  Returns (ok, message)."""
    got_idx = np.asarray(got_idx, dtype=np.int64)
    got_logp = np.asarray(got_logp, dtype=np.float64)
    V = z_row.shape[0]
    if got_idx.min() < 0 or got_idx.max() >= V:
        return False, f"index out of range: {got_idx}"
    if len(set(got_idx.tolist())) != K:
        return False, f"duplicate indices: {got_idx}"
    exact = np.lexsort((np.arange(V), -z_row))[:K]
    for k in range(K):
        if got_idx[k] != exact[k]:
            gap = abs(z_row[got_idx[k]] - z_row[exact[k]])
            if gap >= margin:
                return False, (f"slot {k}: got {got_idx[k]} (z={z_row[got_idx[k]]:.6f}) "
                               f"want {exact[k]} (z={z_row[exact[k]]:.6f}), gap {gap:.2e}")
    ref = z_row[got_idx] - lse
    err = np.abs(ref - got_logp).max()
    if not err <= logp_tol:
        return False, f"logp error {err:.3e} > {logp_tol}"
    return True, ""
