"""Seeded synthetic inputs for the block-draft hot path.

This module is the only code shared by the CPU oracle side (tests, the CPU
baseline) and the CUDA side (bench, binding tests). It draws random numbers and
rounds them to bf16 storage; it holds none of the method's arithmetic (no
convolution, no projection, no softmax, no selection, no verification).

Workload shapes follow the drafters described in "DFlash 2: Keep Drafting
Parallel": blocks of 4 to 16 positions (section "a lightweight local
convolution"), a Qwen3-4B-class drafter (hidden 2560) and a 27B-class one
(hidden 5120) over a ~152K vocabulary, plus a small case and a throughput case.

Every array comes from its own child stream of ``np.random.SeedSequence(seed)``
(one child per array name, in the fixed order of ``STREAMS``), so any array can
be drawn alone and reproduced bit for bit without drawing the others.

bf16 arrays are returned as ``np.uint16`` bit patterns (round-to-nearest-even
from fp32).  "N(0, x)" in the workload recipes names the variance x.
"""
from __future__ import annotations

import dataclasses
import numpy as np

K_TOP = 16

# Order of the per-array child streams; fixed so every array is reproducible.
STREAMS = ("H", "W", "a0", "a1", "x_conv", "prev", "E", "M", "noise", "bonus",
           "topk", "verify", "Wc", "gate", "anchor", "u_walk", "u_accept", "u_resample", "z_target",
           "Pab", "Pg")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int          # blocks
    L: int          # drafted positions per block
    P: int          # positions in the conv input per block
    d: int          # hidden size
    V: int          # vocabulary size
    r: int          # selector rank
    sigma: float    # std of the noise added to h to make the target's tokens
    seed: int
    K: int = K_TOP

    @property
    def M(self) -> int:
        return self.B * self.L


# The five workloads.  P is the conv length: given as [64,8,2560] and
# [256,16,4096] for the batched and throughput cases; elsewhere it is L+1
# (an anchor plus L drafted positions, as in "num-draft-tokens 8" with
# "num_speculative_tokens 7").
WORKLOADS = (
    Workload("tiny", B=1, L=4, P=5, d=256, V=4096, r=32, sigma=0.3, seed=0),
    Workload("qwen3-4b-bs1", B=1, L=7, P=8, d=2560, V=151936, r=64, sigma=0.3, seed=1),
    Workload("qwen3-4b-batched", B=64, L=7, P=8, d=2560, V=151936, r=64, sigma=0.3, seed=2),
    Workload("27b-class", B=16, L=5, P=6, d=5120, V=151936, r=64, sigma=0.5, seed=3),
    Workload("throughput", B=256, L=16, P=16, d=4096, V=129280, r=128, sigma=0.3, seed=4),
)


def workload(i_or_name) -> Workload:
    if isinstance(i_or_name, int):
        return WORKLOADS[i_or_name]
    for w in WORKLOADS:
        if w.name == i_or_name:
            return w
    raise KeyError(i_or_name)


def rng_for(seed: int, stream: str) -> np.random.Generator:
    """Independent PCG64 stream for one named array of one seed."""
    children = np.random.SeedSequence(seed).spawn(len(STREAMS))
    return np.random.Generator(np.random.PCG64(children[STREAMS.index(stream)]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact widening)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float, chunk_rows: int = 8192) -> np.ndarray:
    """N(0, std^2) drawn in fp32, stored as bf16 bits; drawn in row chunks so
    large tables never need a full fp32 copy."""
    shape = tuple(shape)
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(shape[0], -1)
    cols = flat.shape[1]
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        flat[r0:r1] = f32_to_bf16_bits(x)
    return out


def _uniform_bf16(rng, shape, lo, hi) -> np.ndarray:
    x = rng.uniform(lo, hi, size=shape).astype(np.float32)
    return f32_to_bf16_bits(x)


# --- the arrays of one workload ---------------------------------------------

def hidden(w: Workload) -> np.ndarray:
    """Drafted positions' final hidden states H [B*L, d], N(0,1), bf16; row b*L+i."""
    return _normal_bf16(rng_for(w.seed, "H"), (w.M, w.d), 1.0)


def lm_head(w: Workload) -> np.ndarray:
    """LM-head weight W [V, d], N(0, 1/d), bf16, row-major (K-major)."""
    return _normal_bf16(rng_for(w.seed, "W"), (w.V, w.d), 1.0 / np.sqrt(w.d))


def conv_taps(w: Workload):
    """Base taps a0 ~ U(0.5,1), a1 ~ U(0,0.5), each [d] bf16."""
    a0 = _uniform_bf16(rng_for(w.seed, "a0"), (w.d,), 0.5, 1.0)
    a1 = _uniform_bf16(rng_for(w.seed, "a1"), (w.d,), 0.0, 0.5)
    return a0, a1


def conv_input(w: Workload):
    """Conv input x [B, P, d] and the last verified token's representation
    prev [B, d]; both N(0,1) bf16."""
    x = _normal_bf16(rng_for(w.seed, "x_conv"), (w.B, w.P, w.d), 1.0)
    prev = _normal_bf16(rng_for(w.seed, "prev"), (w.B, w.d), 1.0)
    return x, prev


def conv_correction(w: Workload, scale: float = 0.05) -> np.ndarray:
    """Dynamic-conv correction projection Wc [2*d/16, d] bf16: rows 0..d/16-1
    map the hidden state to tap-0 corrections of the 16-channel groups, the
    rest to tap-1 corrections.  N(0, (scale^2)/d), so a correction is about
    N(0, scale^2) for unit-variance inputs ("a small correction")."""
    return _normal_bf16(rng_for(w.seed, "Wc"), (2 * (w.d // 16), w.d), scale / np.sqrt(w.d))


def selector_tables(w: Workload, scale: float = 1.0):
    """Selector stand-in tables E [V, r] and M [r, r], N(0, 0.1) bf16.
    ``scale`` multiplies both standard deviations (tests use it to move
    between the 'selector ~ top-1' and 'pair term dominates' regimes)."""
    std = np.sqrt(0.1) * scale
    E = _normal_bf16(rng_for(w.seed, "E"), (w.V, w.r), std)
    M = _normal_bf16(rng_for(w.seed, "M"), (w.r, w.r), std)
    return E, M


def target_hidden(w: Workload, H_bits: np.ndarray | None = None) -> np.ndarray:
    """Hidden states whose argmax through W gives the target's tokens.

    Rows b*(L+1)+i for i<L hold bf16(h_{b,i} + sigma*n), the drafted hidden
    state plus Gaussian noise; row b*(L+1)+L holds bf16(n') (the bonus position,
    which the drafter does not draft).  Shape [B*(L+1), d] bf16."""
    if H_bits is None:
        H_bits = hidden(w)
    h = bf16_bits_to_f32(H_bits).reshape(w.B, w.L, w.d)
    n = rng_for(w.seed, "noise").standard_normal((w.B, w.L, w.d), dtype=np.float32)
    bonus = rng_for(w.seed, "bonus").standard_normal((w.B, 1, w.d), dtype=np.float32)
    rows = np.concatenate([h + np.float32(w.sigma) * n, bonus], axis=1)
    return f32_to_bf16_bits(rows.reshape(w.B * (w.L + 1), w.d))


# --- stage-level inputs for the selector and verification --------------------

def synthetic_topk(B: int, L: int, V: int, seed: int, K: int = K_TOP, spread: float = 1.0):
    """A stand-alone top-K candidate list: logp [B*L, K] fp32, non-increasing
    and <= 0 along each row, and idx [B*L, K] int32, distinct within a row."""
    rng = rng_for(seed, "topk")
    steps = rng.exponential(spread, size=(B * L, K)).astype(np.float32)
    logp = -np.cumsum(steps, axis=1).astype(np.float32)
    idx = np.empty((B * L, K), dtype=np.int32)
    for m in range(B * L):
        idx[m] = rng.choice(V, size=K, replace=False)
    return logp, idx


def synthetic_verify(B: int, L: int, V: int, seed: int, p_match):
    """Draft tokens [B, L] and target tokens [B, L+1] (int32) where position i
    of the target equals the draft with probability p_match[i], independently
    per position; otherwise it is a different token."""
    rng = rng_for(seed, "verify")
    p = np.broadcast_to(np.asarray(p_match, dtype=np.float64), (L,))
    draft = rng.integers(0, V, size=(B, L), dtype=np.int64)
    hit = rng.random((B, L)) < p[None, :]
    other = (draft + rng.integers(1, V, size=(B, L))) % V
    target = np.empty((B, L + 1), dtype=np.int64)
    target[:, :L] = np.where(hit, draft, other)
    target[:, L] = rng.integers(0, V, size=B)
    return draft.astype(np.int32), target.astype(np.int32)


# --- inputs of the sampled walk and of rejection-sampling verification -------

def anchors(B: int, V: int, seed: int) -> np.ndarray:
    """The last verified token of each block, uniform over [0, V), int32 [B]."""
    return rng_for(seed, "anchor").integers(0, V, size=B).astype(np.int32)


def uniforms(shape, seed: int, stream: str) -> np.ndarray:
    """fp32 uniforms in [0, 1) for one of the named draws ("u_walk",
    "u_accept", "u_resample")."""
    if stream not in ("u_walk", "u_accept", "u_resample"):
        raise KeyError(stream)
    u = rng_for(seed, stream).random(size=shape, dtype=np.float32)
    return np.minimum(u, np.float32(1.0 - 2.0 ** -24))


def target_logits(rows: int, V: int, seed: int, scale: float = 2.0) -> np.ndarray:
    """A target model's logits for `rows` positions: fp32 N(0, scale^2) [rows, V]."""
    rng = rng_for(seed, "z_target")
    out = np.empty((rows, V), dtype=np.float32)
    for r0 in range(0, rows, 64):
        r1 = min(rows, r0 + 64)
        out[r0:r1] = rng.standard_normal((r1 - r0, V), dtype=np.float32) * np.float32(scale)
    return out


def ctx_scorer_weights(w: Workload, e: int = 256, scale: float = 0.2):
    """Weights of the context-gated pair scorer: Pab [2e, d] ~ N(0, scale^2)
    (the A and B projections of a token embedding; with the tied embedding
    table = the LM head, N(0, 1/d), A and B are about N(0, scale^2)) and the
    gate projection Pg [e, d] ~ N(0, 1/d) (a gate input of about N(0, 1) for
    unit-variance hidden states).  bf16."""
    Pab = _normal_bf16(rng_for(w.seed, "Pab"), (2 * e, w.d), scale)
    Pg = _normal_bf16(rng_for(w.seed, "Pg"), (e, w.d), 1.0 / np.sqrt(w.d))
    return Pab, Pg
