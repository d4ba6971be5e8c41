// Path selection: pair scores of neighbouring candidates + max-sum walk.
//
// "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
// every adjacent candidate pair is scored at once and the only serial part is
// one walk over the precomputed scores.  Scorer (a seeded stand-in for the
// pages' trained one, same shape: unary drafter term + low-rank bilinear
// pair term):
//   S_i[j,k] = lp[i,j] + lp[i+1,k] + (e_{c_ij} M) . e_{c_{i+1,k}}
// Walk: delta_0 = 0, delta_{i+1}[k] = max_j delta_i[j] + S_i[j,k] (ties: lowest
// j), end at argmax_k delta_{L-1}[k] (ties: lowest k), then backtrack.
//
// One CTA per block (1024 threads when there are few blocks, else 256):
//   1. gather the 16*L candidate rows of E and the matrix M into shared memory
//      (bf16, rows padded by 16 bytes so 16-byte loads of 8 neighbouring rows
//      hit distinct banks);
//   2. u_ij = e_{c_ij} M for all candidates of a chunk of positions (fp32),
//      then the 16x16 pair scores of those positions, one (j,k) per thread;
//   3. warp 0 walks the scores: lane (h,k) takes the max over j in half h of
//      delta[j] + S[j,k], one xor-16 shuffle joins the halves, backpointers
//      go to shared memory; then a 16-lane argmax and a backtrack.
#include "common.cuh"

namespace dflash {
namespace sel {

constexpr int MAX_THREADS = 1024;
constexpr int KC = 16;
constexpr int U_BUDGET = 48 * 1024;

struct Layout {
  int rp;        // padded E row length (bf16)
  int up;        // padded u row length (fp32)
  int pc;        // positions per u chunk
  size_t m_off, e_off, u_off, s_off, lp_off, tok_off, bp_off, total;
};

__host__ __device__ inline Layout layout(int L, int r) {
  Layout o;
  o.rp = r + 8;
  o.up = r + 4;
  const int npos = L > 1 ? L - 1 : 1;
  int pc = U_BUDGET / (KC * o.up * 4);
  if (pc < 1) pc = 1;
  if (pc > npos) pc = npos;
  o.pc = pc;
  size_t off = 0;
  o.m_off = off;
  off += static_cast<size_t>(r) * r * 2;
  off = (off + 15) & ~size_t(15);
  o.e_off = off;
  off += static_cast<size_t>(L) * KC * o.rp * 2;
  off = (off + 15) & ~size_t(15);
  o.u_off = off;
  off += static_cast<size_t>(pc) * KC * o.up * 4;
  o.s_off = off;
  off += static_cast<size_t>(npos) * KC * KC * 4;
  o.lp_off = off;
  off += static_cast<size_t>(L) * KC * 4;
  o.tok_off = off;
  off += static_cast<size_t>(L) * KC * 4;
  o.bp_off = off;
  off += static_cast<size_t>(npos) * KC;
  o.total = (off + 15) & ~size_t(15);
  return o;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(MAX_THREADS) path_select_kernel(
    const float* __restrict__ topk_logp, const int32_t* __restrict__ topk_idx, const uint16_t* __restrict__ E,
    const uint16_t* __restrict__ Msel, int L, int r, int V, int32_t* __restrict__ path_tok,
    int32_t* __restrict__ path_slot, float* __restrict__ path_score, float* __restrict__ pair_dbg, int* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  const Layout lo = layout(L, r);
  uint16_t* Ms = reinterpret_cast<uint16_t*>(smem + lo.m_off);
  uint16_t* Es = reinterpret_cast<uint16_t*>(smem + lo.e_off);
  float* Us = reinterpret_cast<float*>(smem + lo.u_off);
  float* Ss = reinterpret_cast<float*>(smem + lo.s_off);
  float* lps = reinterpret_cast<float*>(smem + lo.lp_off);
  int* toks = reinterpret_cast<int*>(smem + lo.tok_off);
  int8_t* bps = reinterpret_cast<int8_t*>(smem + lo.bp_off);

  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  const int r8 = r / 8;
  const size_t row0 = static_cast<size_t>(b) * L;

  // ---- 1. candidates, their E rows, and M into shared memory -------------
  for (int q = tid; q < L * KC; q += nthr) {
    lps[q] = topk_logp[row0 * KC + q];
    int c = topk_idx[row0 * KC + q];
    if (c < 0 || c >= V) {
      set_status(status, DFLASH_ERR_BAD_INDEX);
      c = 0;
    }
    toks[q] = c;
  }
  {
    const uint4* Mg = reinterpret_cast<const uint4*>(Msel);
    uint4* Mv = reinterpret_cast<uint4*>(Ms);
    for (int q = tid; q < r * r8; q += nthr) Mv[q] = __ldg(Mg + q);
  }
  __syncthreads();
  for (int q = tid; q < L * KC * r8; q += nthr) {
    const int cand = q / r8;
    const int v8 = q - cand * r8;
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(E + static_cast<size_t>(toks[cand]) * r) + v8);
    *reinterpret_cast<uint4*>(Es + static_cast<size_t>(cand) * lo.rp + v8 * 8) = val;
  }
  __syncthreads();

  // ---- 2. pair scores, a chunk of positions at a time --------------------
  const int npos = L - 1;
  for (int i0 = 0; i0 < npos; i0 += lo.pc) {
    const int pcn = min(lo.pc, npos - i0);
    // u[ii][j][t] = sum_s e_{c_(i0+ii),j}[s] * M[s][t], 8 outputs per item
    for (int q = tid; q < pcn * KC * r8; q += nthr) {
      const int tg = q % r8;
      const int jj = q / r8;  // (ii * 16 + j)
      const int ii = jj / KC;
      const int j = jj - ii * KC;
      const uint16_t* er = Es + static_cast<size_t>((i0 + ii) * KC + j) * lo.rp;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < r; ++s) {
        const float es = __uint_as_float(static_cast<uint32_t>(er[s]) << 16);
        const uint4 mv = *reinterpret_cast<const uint4*>(Ms + static_cast<size_t>(s) * r + tg * 8);
        acc[0] = fmaf(es, bf_lo(mv.x), acc[0]);
        acc[1] = fmaf(es, bf_hi(mv.x), acc[1]);
        acc[2] = fmaf(es, bf_lo(mv.y), acc[2]);
        acc[3] = fmaf(es, bf_hi(mv.y), acc[3]);
        acc[4] = fmaf(es, bf_lo(mv.z), acc[4]);
        acc[5] = fmaf(es, bf_hi(mv.z), acc[5]);
        acc[6] = fmaf(es, bf_lo(mv.w), acc[6]);
        acc[7] = fmaf(es, bf_hi(mv.w), acc[7]);
      }
      float* ur = Us + static_cast<size_t>(jj) * lo.up + tg * 8;
      *reinterpret_cast<float4*>(ur) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(ur + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    __syncthreads();
    for (int q = tid; q < pcn * KC * KC; q += nthr) {
      const int k = q % KC;
      const int j = (q / KC) % KC;
      const int ii = q / (KC * KC);
      const int i = i0 + ii;
      const float* ur = Us + static_cast<size_t>(ii * KC + j) * lo.up;
      const uint16_t* er = Es + static_cast<size_t>((i + 1) * KC + k) * lo.rp;
      float acc = 0.f;
      for (int t = 0; t < r; t += 8) {
        const float4 u0 = *reinterpret_cast<const float4*>(ur + t);
        const float4 u1 = *reinterpret_cast<const float4*>(ur + t + 4);
        const uint4 ev = *reinterpret_cast<const uint4*>(er + t);
        acc = fmaf(u0.x, bf_lo(ev.x), acc);
        acc = fmaf(u0.y, bf_hi(ev.x), acc);
        acc = fmaf(u0.z, bf_lo(ev.y), acc);
        acc = fmaf(u0.w, bf_hi(ev.y), acc);
        acc = fmaf(u1.x, bf_lo(ev.z), acc);
        acc = fmaf(u1.y, bf_hi(ev.z), acc);
        acc = fmaf(u1.z, bf_lo(ev.w), acc);
        acc = fmaf(u1.w, bf_hi(ev.w), acc);
      }
      const float sc = (lps[i * KC + j] + lps[(i + 1) * KC + k]) + acc;
      Ss[(i * KC + j) * KC + k] = sc;
      if (pair_dbg) pair_dbg[((static_cast<size_t>(b) * npos + i) * KC + j) * KC + k] = sc;
    }
    __syncthreads();
  }

  // ---- 3. max-sum walk (warp 0) -------------------------------------------
  if (tid < 32) {
    const int lane = tid;
    const int k = lane & 15;
    const int h = lane >> 4;
    float delta = 0.f;  // lanes k and 16+k both hold delta[k]
    for (int i = 0; i < npos; ++i) {
      float best = -INFINITY;
      int bj = 0;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = h * 8 + jj;
        const float dj = __shfl_sync(0xffffffffu, delta, j);
        const float val = dj + Ss[(i * KC + j) * KC + k];
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
      if (h == 0) bps[i * KC + k] = static_cast<int8_t>(bj);
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
    if (lane == 0) {
      int slot = npos > 0 ? bk : 0;
      const float score = npos > 0 ? bv : 0.f;
      for (int i = L - 1; i >= 0; --i) {
        path_tok[row0 + i] = toks[i * KC + slot];
        if (path_slot) path_slot[row0 + i] = slot;
        if (i > 0) slot = bps[(i - 1) * KC + slot];
      }
      if (path_score) path_score[b] = score;
    }
  }
}

}  // namespace sel
}  // namespace dflash

extern "C" int dflash_path_select(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                                  const dflash_bf16* Msel, int B, int L, int K, int r, int V, int32_t* path_tok,
                                  int32_t* path_slot, float* path_score, float* pair_scores_dbg, int* dev_status,
                                  void* stream) {
  using namespace dflash::sel;
  if (!topk_logp || !topk_idx || !E || !Msel || !path_tok) return DFLASH_ERR_INVALID_ARG;
  if (K != KC || B < 1 || L < 1 || L > 16 || r < 8 || r > 128 || r % 8 != 0 || V < 1)
    return DFLASH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(E) | reinterpret_cast<uintptr_t>(Msel)) & 15) return DFLASH_ERR_INVALID_ARG;
  const Layout lo = layout(L, r);
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(path_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) !=
        cudaSuccess)
      return DFLASH_ERR_CUDA;
    attr_done = true;
  }
  // Few blocks: spread each block's candidate work over more threads (latency);
  // many blocks: 256 threads so several CTAs share an SM.
  const int threads = B < 128 ? 1024 : 256;
  path_select_kernel<<<B, threads, lo.total, static_cast<cudaStream_t>(stream)>>>(
      topk_logp, topk_idx, E, Msel, L, r, V, path_tok, path_slot, path_score, pair_scores_dbg, dev_status);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
