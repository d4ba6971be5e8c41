// Serial walks over pair-score tables in shared memory (one warp).
//
// "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
// scoring is parallel; the only serial part is one walk over the
// precomputed scores.  Tables: internal positions 0..T, table i holds
// S_i[j][k] at Ss[(i*16 + j)*16 + k] (row j = slot at internal position i,
// column k = slot at internal position i+1); toks[p*16 + j] is the token of
// slot j at internal position p.  Internal position OFF + p is drafted
// position p (OFF = 1 when internal position 0 is the last verified token,
// whose 16 rows are copies).
#pragma once

#include "common.cuh"

namespace dflash {
namespace walk {

constexpr int WKC = 16;

enum Walk { WALK_VITERBI = 0, WALK_GREEDY = 1, WALK_SAMPLE = 2 };

struct WalkArgs {
  const int32_t* anchor;   // [B] last verified token (greedy / sample)
  const float* uniforms;   // [B, L] one uniform per drafted position (sample)
  float inv_t;             // 1 / temperature (sample)
  float* path_q;           // [B, L, 16] distribution each slot was drawn from (nullable)
};

// Max-sum (Viterbi) walk over T tables: delta_0 = 0; delta_{i+1}[k] =
// max_j delta_i[j] + S_i[j][k] (ties: lowest j); the end is argmax_k delta_T
// (ties: lowest k), then a backtrack.  Lane (h, k) maximises over the 8
// predecessors of half h, an xor-16 shuffle joins the halves, backpointers
// go to bps (int8); pslot receives the slot of every internal position.
// Writes drafted positions 0..L-1; path_score = delta_T at the end (0 when
// T = 0).  verify: lane i holds the target token i in pre_t.
__device__ __forceinline__ void walk_maxsum(const float* Ss, const int* toks, int T, int OFF, int L, int b,
                                            int8_t* bps, int* pslot, int pre_t, int32_t* path_tok,
                                            int32_t* path_slot, float* path_score, bool verify,
                                            int32_t* accept_len, int32_t* next_token) {
  const int lane = threadIdx.x & 31;
  const int k = lane & 15;
  const int h = lane >> 4;
  const size_t row0 = static_cast<size_t>(b) * L;
  float delta = 0.f;  // lanes k and 16+k both hold delta[k]
  for (int i = 0; i < T; ++i) {
    float best = -INFINITY;
    int bj = 0;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = h * 8 + jj;
      const float dj = __shfl_sync(0xffffffffu, delta, j);
      const float val = dj + Ss[(i * WKC + j) * WKC + k];
      if (val > best) {
        best = val;
        bj = j;
      }
    }
    const float ob = __shfl_xor_sync(0xffffffffu, best, 16);
    const int oj = __shfl_xor_sync(0xffffffffu, bj, 16);
    // prefer the lower half (lower j) on ties
    const bool take = h == 0 ? (ob > best) : (ob >= best);
    if (take) {
      best = ob;
      bj = oj;
    }
    delta = best;
    if (h == 0) bps[i * WKC + k] = static_cast<int8_t>(bj);
  }
  __syncwarp();
  // argmax over k (lanes 0..15), ties to the lowest k
  float bv = delta;
  int bk = k;
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, bv, off);
    const int k2 = __shfl_xor_sync(0xffffffffu, bk, off);
    if (v2 > bv || (v2 == bv && k2 < bk)) {
      bv = v2;
      bk = k2;
    }
  }
  // backtrack (lane 0), then lane p writes drafted position p
  if (lane == 0) {
    int slot = T > 0 ? bk : 0;
    for (int i = T; i >= 0; --i) {
      pslot[i] = slot;
      if (i > 0) slot = bps[(i - 1) * WKC + slot];
    }
    if (path_score) path_score[b] = T > 0 ? bv : 0.f;
  }
  __syncwarp();
  const bool in_block = lane < L;
  const int my_slot = in_block ? pslot[lane + OFF] : 0;
  const int my_tok = in_block ? toks[(lane + OFF) * WKC + my_slot] : 0;
  if (in_block) {
    path_tok[row0 + lane] = my_tok;
    if (path_slot) path_slot[row0 + lane] = my_slot;
  }
  if (verify) {
    const bool differs = in_block && my_tok != pre_t;
    const unsigned mask = __ballot_sync(0xffffffffu, differs);
    const int n = mask ? __ffs(mask) - 1 : L;
    const int nt = __shfl_sync(0xffffffffu, pre_t, n);
    if (lane == 0) {
      accept_len[b] = n + 1;
      next_token[b] = nt;
    }
  }
}

// One warp walks L steps from the anchor over the pair tables in shared
// memory (table i: row = previous slot, column = next slot).  Lane (h, k)
// holds column k; both half-warps compute the same values.
//   greedy: next = argmax_k S_i[cur, k] (ties: lowest k)
//   sample: q = softmax(S_i[cur, :] / T); next = the smallest k whose
//           cumulative q exceeds u_i (inverse CDF in slot order)
// pre_t / pre_u: lane i holds target token i / uniform i (read earlier).
template <int WALK>
__device__ __forceinline__ void walk_from_anchor(const float* Ss, const int* toks, int L, int b, const WalkArgs& wa,
                                                 int pre_t, float pre_u, int32_t* path_tok, int32_t* path_slot,
                                                 float* path_score, bool verify, int32_t* accept_len,
                                                 int32_t* next_token) {
  const int lane = threadIdx.x & 31;
  const int k = lane & 15;
  const size_t row0 = static_cast<size_t>(b) * L;
  int cur = 0;
  int my_slot = 0;  // lane i keeps the slot chosen at position i
  float score = 0.f;
  for (int i = 0; i < L; ++i) {
    const float v = Ss[(i * WKC + cur) * WKC + k];
    int nk;
    if (WALK == WALK_GREEDY) {
      float bv = v;
      int bk = k;
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, bv, off);
        const int k2 = __shfl_xor_sync(0xffffffffu, bk, off);
        if (v2 > bv || (v2 == bv && k2 < bk)) {
          bv = v2;
          bk = k2;
        }
      }
      nk = bk;
    } else {
      float m = v;
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float e = expf((v - m) * wa.inv_t);
      // inclusive prefix sum over the 16 lanes of each half
      float c = e;
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, c, off, 16);
        if (k >= off) c += t;
      }
      const float total = __shfl_sync(0xffffffffu, c, 15);
      const float u = __shfl_sync(0xffffffffu, pre_u, i);
      const unsigned over = __ballot_sync(0xffffffffu, c > u * total) & 0xffffu;
      nk = over ? __ffs(over) - 1 : 15;
      if (wa.path_q && lane < 16) wa.path_q[(row0 + i) * WKC + k] = e / total;
    }
    score += __shfl_sync(0xffffffffu, v, nk);
    if (lane == i) my_slot = nk;
    cur = nk;
  }
  const bool in_block = lane < L;
  const int my_tok = in_block ? toks[(lane + 1) * WKC + my_slot] : 0;
  if (in_block) {
    path_tok[row0 + lane] = my_tok;
    if (path_slot) path_slot[row0 + lane] = my_slot;
  }
  if (path_score && lane == 0) path_score[b] = score;
  if (verify) {
    const bool differs = in_block && my_tok != pre_t;
    const unsigned mask = __ballot_sync(0xffffffffu, differs);
    const int n = mask ? __ffs(mask) - 1 : L;
    const int nt = __shfl_sync(0xffffffffu, pre_t, n);
    if (lane == 0) {
      accept_len[b] = n + 1;
      next_token[b] = nt;
    }
  }
}

}  // namespace walk
}  // namespace dflash
