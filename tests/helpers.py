"""Test-side helpers: move seeded inputs to the GPU, compare with the oracle."""
import numpy as np
import torch

import oracle


def dev_bf16(bits):
    import block_draft_selection_b200 as bds
    return bds.bf16_tensor(bits, "cuda")


def to_np(t):
    return t.detach().cpu().numpy()


def bf16_out_to_f64(t):
    """torch bf16 tensor -> float64 numpy (exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def logits_bound(H_bits, W_bits, rows=None):
    """A priori bound on |fp32-accumulated z - exact z| per (row, v):
    4 * d * 2^-23 * sum_k |H[m,k] W[v,k]| + 1e-6 (products of bf16 values are
    exact in fp32; each of the d accumulations adds at most one fp32 rounding,
    with slack for an accumulation order and rounding mode we do not control)."""
    from block_draft_synth import bf16_bits_to_f32
    H = np.abs(bf16_bits_to_f32(H_bits).astype(np.float64))
    if rows is not None:
        H = H[rows]
    W = np.abs(bf16_bits_to_f32(W_bits).astype(np.float64))
    d = H.shape[1]
    return 4 * d * 2.0 ** -23 * (H @ W.T) + 1e-6


def check_topk_rows(z, lse, got_idx, got_logp, rows=None, margin=1e-3, tol=2e-2):
    """Every listed row of the GPU output passes the margin-aware comparison."""
    rows = range(z.shape[0]) if rows is None else rows
    bad = []
    for n, m in enumerate(rows):
        ok, msg = oracle.topk_margin_ok(z[n], lse[n], got_idx[m], got_logp[m], 16, margin, tol)
        if not ok:
            bad.append((m, msg))
    assert not bad, bad[:5]


def exact_ties_free(z_row, K=16, margin=1e-3):
    s = np.sort(z_row)[::-1][:K + 1]
    return np.min(np.abs(np.diff(s))) >= margin
