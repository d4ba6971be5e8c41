"""CPU oracle for the block-draft hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct float64 restatement of what the path
computes, written from the DFlash 2 pages ("DFlash 2: Keep Drafting Parallel",
the Chinese translation of the blog, and "Inco AI's DFlash 2 lifts LLM decoding
output 16-25%") plus the stand-in scorer and walk that this library fixes where
the pages leave the computation open.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or run anything here.  The CUDA library never calls
it, shares no code with it, and has no CPU fallback.

Inputs are the same bf16 bit patterns (np.uint16) the GPU path receives; the
oracle widens them exactly to float64 and computes the plain definitions with
no blocking, fusion or reordering beyond what each definition states.

Pins (``tests/test_oracle_*.py``, run with ``-m "not gpu"``):
  conv2tap      hand-worked case, identity/shift taps, marker inputs
  conv2tap_dynamic
                zero correction = the static conv, a hand-worked case, a
                correction confined to its 16-channel group
  lmhead_topk   exact rational/decimal brute force on tiny shapes, heap
                selection, the uniform-logit case (lse = log V)
  argmax_tokens exact brute force, tie to the lowest index
  pair_scores / viterbi / path_select
                exhaustive 16^L enumeration for L <= 4 on an exact rational
                pair table, the E = 0 case (= the top-1 path), a hand case
  verify        hand cases and the Table 1 closed form (4.27 / 6.79)
  greedy_walk / sample_walk
                a hand case where greedy misses the anchored max-sum path,
                exact rational scores on random tiny cases, the T -> 0 limit
                (= greedy), the E = 0 closed form at T = 1 (the renormalised
                top-16), and the path distribution integrated over a grid of
                uniforms against exact conditional softmaxes
  ctx_tables / ctx_select (the pages' context-gated scorer)
                a hand-worked case, exact rational tables with the gate
                fixed at 1/2 and at 1, brute force over all 16^L anchored
                paths, zero projections (= top-1 path), a planted swap of
                the two projections
  verify_rejection
                hand cases, and the output-distribution theorem: the first
                emitted token is distributed exactly as the target's p_0
                (integrated over grids of both uniforms)
"""
from .conv import conv2tap, conv2tap_dynamic
from .lmhead import logits, lmhead_topk, argmax_tokens, topk_margin_ok
from .selector import pair_scores, viterbi, viterbi_two_best, path_select
from .verify import verify
from .ctx_scorer import ctx_tables, ctx_select, maxsum_walk_tables
from .walks import anchor_scores, greedy_walk, sample_walk, verify_rejection, inverse_cdf, target_probs

__all__ = ["conv2tap", "conv2tap_dynamic", "logits", "lmhead_topk", "argmax_tokens", "topk_margin_ok",
           "pair_scores", "viterbi", "viterbi_two_best", "path_select", "verify",
           "anchor_scores", "greedy_walk", "sample_walk", "verify_rejection", "inverse_cdf",
           "target_probs", "ctx_tables", "ctx_select", "maxsum_walk_tables"]
