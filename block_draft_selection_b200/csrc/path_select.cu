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
// One thread-block cluster of Q CTAs per block; Q = 1 (one CTA of 512
// threads) when there are enough blocks to fill the GPU, else up to 8 CTAs of
// 256 threads so that a block's pair scoring spreads over Q SMs:
//   1. each CTA gathers the E rows of the positions it scores and the matrix
//      M into shared memory (bf16, rows padded by 16 bytes so 16-byte loads
//      of 8 neighbouring rows hit distinct banks);
//   2. CTA q scores position pairs i = q, q+Q, ...: u_ij = e_{c_ij} M on the
//      tensor cores (mma.sync m16n8k16, bf16 in, fp32 out; M staged
//      transposed; r not a multiple of 16 falls back to CUDA-core FMAs), then
//      the 16x16 pair scores in fp32, one (j,k) per thread, written straight
//      into the leader CTA's shared memory (distributed shared memory);
//   3. after a cluster barrier, warp 0 of the leader walks the scores
//      (walk.cuh): lane (h,k) takes the max over j in half h of
//      delta[j] + S[j,k], one xor-16 shuffle joins the halves, backpointers
//      go to shared memory; then a 16-lane argmax, a backtrack and
//      (optionally) greedy verification against target tokens read at the
//      start.
//
// The same kernel also walks from the last verified ("anchor") token, the
// walk the section describes: greedily following the best successor, or
// drawing each successor from softmax(score / T) over the 16 candidates.
// For these walks an extra internal position 0 holds the anchor (16 copies
// of its E row, log-probability 0), so the first pair table is
//   S_a[k] = lp[0,k] + (e_anchor M) . e_{c_0k}
// and internal position p >= 1 is drafted position p - 1.
#include <cstdlib>
#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
#include "walk.cuh"

namespace dflash {
namespace sel {

constexpr int THREADS = 512;         // launch bound: 512 per CTA when Q = 1
constexpr int THREADS_CLUSTER = 256; // per CTA of a cluster (Q > 1)
constexpr int MAX_CLUSTER = 8;
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
  off += static_cast<size_t>(r) * o.rp * 2;  // M, or its transpose with padded rows (tensor-core path)
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

// d += A (16x16, row-major, bf16) . B (16x8, column-major, bf16), fp32
// accumulate; fragments in the standard m16n8k16 register layout.
__device__ __forceinline__ void mma_bf16_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

using namespace walk;

template <int WALK>
__global__ void __launch_bounds__(THREADS) path_select_kernel(
    const float* __restrict__ topk_logp, const int32_t* __restrict__ topk_idx, const uint16_t* __restrict__ E,
    const uint16_t* __restrict__ Msel, int L, int r, int V, int32_t* __restrict__ path_tok,
    int32_t* __restrict__ path_slot, float* __restrict__ path_score, float* __restrict__ pair_dbg, int* status,
    const int32_t* __restrict__ target, int32_t* __restrict__ accept_len, int32_t* __restrict__ next_token, int Q,
    WalkArgs wa) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int OFF = WALK == WALK_VITERBI ? 0 : 1;  // internal positions before drafted position 0
  const int Li = L + OFF;                            // internal positions
  const Layout lo = layout(Li, r);
  uint16_t* Ms = reinterpret_cast<uint16_t*>(smem + lo.m_off);
  uint16_t* Es = reinterpret_cast<uint16_t*>(smem + lo.e_off);
  float* Us = reinterpret_cast<float*>(smem + lo.u_off);
  float* Ss = reinterpret_cast<float*>(smem + lo.s_off);
  float* lps = reinterpret_cast<float*>(smem + lo.lp_off);
  int* toks = reinterpret_cast<int*>(smem + lo.tok_off);
  int8_t* bps = reinterpret_cast<int8_t*>(smem + lo.bp_off);

  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x / Q;
  const int q_rank = blockIdx.x - b * Q;  // rank in the cluster (clusters are Q consecutive CTAs)
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  const int r8 = r / 8;
  const size_t row0 = static_cast<size_t>(b) * L;
  const int npos = Li - 1;  // pair tables
  // The leader's warp 0 reads now what the walk and the verification need at
  // the end (lane i: target token i, uniform i), so those loads overlap the
  // scoring instead of following the walk.
  int pre_t = 0;
  float pre_u = 0.f;
  if (q_rank == 0 && tid < 32) {
    if (target != nullptr && tid <= L) pre_t = __ldg(target + static_cast<size_t>(b) * (L + 1) + tid);
    if (WALK == WALK_SAMPLE && tid < L) pre_u = __ldg(wa.uniforms + row0 + tid);
  }
  // Scores go to the leader's shared memory (this CTA's own when Q == 1).
  // The leader's shared memory may be written only once every CTA of the
  // cluster runs: arrive now, wait just before the first remote store.
  float* S_out = Ss;
  if (Q > 1) {
    S_out = cooperative_groups::this_cluster().map_shared_rank(Ss, 0);
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  }
  // positions this CTA needs rows for: i and i+1 for every i = q_rank (mod Q)
  auto needs_pos = [&](int i) {
    if (Q == 1) return true;
    const bool as_left = i < npos && (i % Q) == q_rank;
    const bool as_right = i >= 1 && ((i - 1) % Q) == q_rank;
    return as_left || as_right;
  };

  // ---- 1. candidates, their E rows, and M into shared memory -------------
  // One pass: every load here depends only on global inputs, so the index
  // reads, the E-row gathers that follow them and the copy of M are all in
  // flight together.
  int anchor_tok = 0;
  if (OFF) {
    anchor_tok = __ldg(wa.anchor + b);
    if (anchor_tok < 0 || anchor_tok >= V) {
      if (tid == 0) set_status(status, DFLASH_ERR_BAD_INDEX);
      anchor_tok = 0;
    }
  }
  for (int q = tid; q < Li * KC; q += nthr) {
    if (OFF && q < KC) {  // the anchor: 16 copies, no unary term
      lps[q] = 0.f;
      toks[q] = anchor_tok;
      continue;
    }
    lps[q] = __ldg(topk_logp + row0 * KC + (q - OFF * KC));
    int c = __ldg(topk_idx + row0 * KC + (q - OFF * KC));
    if (c < 0 || c >= V) {
      set_status(status, DFLASH_ERR_BAD_INDEX);
      c = 0;
    }
    toks[q] = c;
  }
  const bool use_mma = (r % 16) == 0;
  {
    const uint4* Mg = reinterpret_cast<const uint4*>(Msel);
    if (use_mma) {
      // transposed, rows padded to rp: column t of M is row t here, so the
      // tensor-core B fragments are 32-bit loads without bank conflicts.  A
      // warp moves one 8-column group of 32 consecutive source rows: lane l
      // reads row 32*blk + l and its 16-bit stores land in neighbouring
      // halfwords of each destination row (no bank conflicts, where lanes
      // walking the columns of one row would all hit one bank).
      const int lane = tid & 31, nwarp = nthr >> 5;
      const int nblk = (r + 31) / 32;
      for (int item = tid >> 5; item < r8 * nblk; item += nwarp) {
        const int c8 = item % r8;
        const int srow = (item / r8) * 32 + lane;
        if (srow < r) {
          const uint4 v = __ldg(Mg + static_cast<size_t>(srow) * r8 + c8);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 8; ++e)
            Ms[static_cast<size_t>(c8 * 8 + e) * lo.rp + srow] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
        }
      }
    } else {
      uint4* Mv = reinterpret_cast<uint4*>(Ms);
      for (int q = tid; q < r * r8; q += nthr) Mv[q] = __ldg(Mg + q);
    }
  }
  for (int q = tid; q < Li * KC * r8; q += nthr) {
    const int cand = q / r8;
    const int v8 = q - cand * r8;
    if (!needs_pos(cand / KC)) continue;
    int c = (OFF && cand < KC) ? anchor_tok : __ldg(topk_idx + row0 * KC + (cand - OFF * KC));
    c = (c < 0 || c >= V) ? 0 : c;
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(E + static_cast<size_t>(c) * r) + v8);
    *reinterpret_cast<uint4*>(Es + static_cast<size_t>(cand) * lo.rp + v8 * 8) = val;
  }
  __syncthreads();

  if (Q > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");

  // ---- 2. pair scores, a chunk of this CTA's positions at a time ----------
  // This CTA's positions are i = q_rank + Q*m; chunk index ii counts m.
  const int my_npos = npos > q_rank ? (npos - q_rank + Q - 1) / Q : 0;
  for (int m0 = 0; m0 < my_npos; m0 += lo.pc) {
    const int pcn = min(lo.pc, my_npos - m0);
    // u[ii][j][t] = sum_s e_{c_(i0+ii),j}[s] * M[s][t]
    if (use_mma) {
      // On the tensor cores: for each position, u (16 x r) = E rows (16 x r)
      // . M (r x r) as mma.sync m16n8k16 (bf16 in, fp32 accumulate; the
      // products are exact, as on the CUDA cores).  One warp per (position,
      // 8-column n-tile).
      const int warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
      const int ntiles = r / 8;
      for (int item = warp; item < pcn * ntiles; item += nthr / 32) {
        const int ii = item / ntiles;
        const int nt = item - ii * ntiles;
        const int i = q_rank + Q * (m0 + ii);
        const uint16_t* e0 = Es + static_cast<size_t>(i * KC + gq) * lo.rp + 2 * tq;
        const uint16_t* e8 = e0 + 8 * lo.rp;
        const uint16_t* mt = Ms + static_cast<size_t>(nt * 8 + gq) * lo.rp + 2 * tq;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < r; k0 += 16) {
          const uint32_t a0 = *reinterpret_cast<const uint32_t*>(e0 + k0);
          const uint32_t a1 = *reinterpret_cast<const uint32_t*>(e8 + k0);
          const uint32_t a2 = *reinterpret_cast<const uint32_t*>(e0 + k0 + 8);
          const uint32_t a3 = *reinterpret_cast<const uint32_t*>(e8 + k0 + 8);
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(mt + k0);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(mt + k0 + 8);
          mma_bf16_m16n8k16(d, a0, a1, a2, a3, b0, b1);
        }
        float* u0 = Us + static_cast<size_t>(ii * KC + gq) * lo.up + nt * 8 + 2 * tq;
        *reinterpret_cast<float2*>(u0) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(u0 + 8 * lo.up) = make_float2(d[2], d[3]);
      }
    } else {
    // on the CUDA cores, 8 outputs per item; neighbouring lanes take the two
    // halves of the s range and add them with one shuffle (the item count is
    // a multiple of 32: whole warps iterate)
    const int rh = r / 2;
    for (int q = tid; q < pcn * KC * r8 * 2; q += nthr) {
      const int h = q & 1;
      const int tg = (q >> 1) % r8;
      const int jj = (q >> 1) / r8;  // (ii * 16 + j)
      const int ii = jj / KC;
      const int j = jj - ii * KC;
      const int i = q_rank + Q * (m0 + ii);
      const uint16_t* er = Es + static_cast<size_t>(i * KC + j) * lo.rp + h * rh;
      const uint16_t* mr = Ms + static_cast<size_t>(h * rh) * r + tg * 8;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int s = 0; s < rh; ++s) {
        const float es = __uint_as_float(static_cast<uint32_t>(er[s]) << 16);
        const uint4 mv = *reinterpret_cast<const uint4*>(mr + static_cast<size_t>(s) * r);
        acc[0] = fmaf(es, bf_lo(mv.x), acc[0]);
        acc[1] = fmaf(es, bf_hi(mv.x), acc[1]);
        acc[2] = fmaf(es, bf_lo(mv.y), acc[2]);
        acc[3] = fmaf(es, bf_hi(mv.y), acc[3]);
        acc[4] = fmaf(es, bf_lo(mv.z), acc[4]);
        acc[5] = fmaf(es, bf_hi(mv.z), acc[5]);
        acc[6] = fmaf(es, bf_lo(mv.w), acc[6]);
        acc[7] = fmaf(es, bf_hi(mv.w), acc[7]);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 1);
      if (h == 0) {
        float* ur = Us + static_cast<size_t>(jj) * lo.up + tg * 8;
        *reinterpret_cast<float4*>(ur) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(ur + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
    }
    __syncthreads();
    for (int q = tid; q < pcn * KC * KC; q += nthr) {
      const int k = q % KC;
      const int j = (q / KC) % KC;
      const int ii = q / (KC * KC);
      const int i = q_rank + Q * (m0 + ii);
      const float* ur = Us + static_cast<size_t>(ii * KC + j) * lo.up;
      const uint16_t* er = Es + static_cast<size_t>((i + 1) * KC + k) * lo.rp;
      // four independent accumulators (not one chain of r dependent FMAs)
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
      for (int t = 0; t < r; t += 8) {
        const float4 u0 = *reinterpret_cast<const float4*>(ur + t);
        const float4 u1 = *reinterpret_cast<const float4*>(ur + t + 4);
        const uint4 ev = *reinterpret_cast<const uint4*>(er + t);
        a0 = fmaf(u0.x, bf_lo(ev.x), a0);
        a1 = fmaf(u0.y, bf_hi(ev.x), a1);
        a2 = fmaf(u0.z, bf_lo(ev.y), a2);
        a3 = fmaf(u0.w, bf_hi(ev.y), a3);
        a0 = fmaf(u1.x, bf_lo(ev.z), a0);
        a1 = fmaf(u1.y, bf_hi(ev.z), a1);
        a2 = fmaf(u1.z, bf_lo(ev.w), a2);
        a3 = fmaf(u1.w, bf_hi(ev.w), a3);
      }
      const float acc = (a0 + a1) + (a2 + a3);
      const float sc = (lps[i * KC + j] + lps[(i + 1) * KC + k]) + acc;
      S_out[(i * KC + j) * KC + k] = sc;
      if (WALK == WALK_VITERBI && pair_dbg) pair_dbg[((static_cast<size_t>(b) * npos + i) * KC + j) * KC + k] = sc;
    }
    __syncthreads();
  }

  // ---- 3. max-sum walk (warp 0 of the leader) -----------------------------
  if (Q > 1) {
    cooperative_groups::this_cluster().sync();  // every CTA's scores have landed
    if (q_rank != 0) return;
  }
  if (WALK != WALK_VITERBI) {
    if (tid < 32)
      walk_from_anchor<WALK>(Ss, toks, L, b, wa, pre_t, pre_u, path_tok, path_slot, path_score, target != nullptr,
                             accept_len, next_token);
    return;
  }
  if (tid < 32)
    walk_maxsum(Ss, toks, npos, 0, L, b, bps, reinterpret_cast<int*>(Us), pre_t, path_tok, path_slot, path_score,
                target != nullptr, accept_len, next_token);
}

}  // namespace sel
}  // namespace dflash

namespace dflash {
namespace sel {

template <int WALK>
static int launch(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E, const dflash_bf16* Msel,
                  int B, int L, int K, int r, int V, int32_t* path_tok, int32_t* path_slot, float* path_score,
                  float* pair_scores_dbg, const int32_t* target, int32_t* accept_len, int32_t* next_token,
                  int* dev_status, void* stream, WalkArgs wa) {
  if (!topk_logp || !topk_idx || !E || !Msel || !path_tok) return DFLASH_ERR_INVALID_ARG;
  if (K != KC || B < 1 || L < 1 || L > 16 || r < 8 || r > 128 || r % 8 != 0 || V < 1)
    return DFLASH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(E) | reinterpret_cast<uintptr_t>(Msel)) & 15) return DFLASH_ERR_INVALID_ARG;
  constexpr int OFF = WALK == WALK_VITERBI ? 0 : 1;
  const int npairs = L + OFF - 1;
  const Layout lo = layout(L + OFF, r);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err =
        cudaFuncSetAttribute(path_select_kernel<WALK>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  });
  if (attr_err != cudaSuccess) return DFLASH_ERR_CUDA;
  // Few blocks: one cluster of up to 8 CTAs per block spreads its pair scoring
  // over several SMs (latency); many blocks fill the GPU one CTA per block.
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // DFLASH_SELECT_Q (read at every call) caps Q (1: always one CTA per block)
  int q_cap = MAX_CLUSTER;
  if (const char* ev = std::getenv("DFLASH_SELECT_Q")) {
    const int v = std::atoi(ev);
    if (v >= 1 && v <= MAX_CLUSTER) q_cap = v;
  }
  int Q = 1;
  if (B * 2 < sms && npairs > 1) {
    Q = npairs < q_cap ? npairs : q_cap;
    while (Q > 1 && static_cast<long long>(B) * Q > sms) --Q;
  }
  const cudaError_t e = launch_kernel_cluster(
      path_select_kernel<WALK>, dim3(B * Q), dim3(Q > 1 ? THREADS_CLUSTER : THREADS), lo.total,
      static_cast<cudaStream_t>(stream), Q,
      topk_logp, topk_idx, reinterpret_cast<const uint16_t*>(E), reinterpret_cast<const uint16_t*>(Msel), L, r, V,
      path_tok, path_slot, path_score, pair_scores_dbg, dev_status, target, accept_len, next_token, Q, wa);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

}  // namespace sel
}  // namespace dflash

extern "C" int dflash_path_select(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                                  const dflash_bf16* Msel, int B, int L, int K, int r, int V, int32_t* path_tok,
                                  int32_t* path_slot, float* path_score, float* pair_scores_dbg, int* dev_status,
                                  void* stream) {
  return dflash::sel::launch<dflash::sel::WALK_VITERBI>(topk_logp, topk_idx, E, Msel, B, L, K, r, V, path_tok,
                                                        path_slot, path_score, pair_scores_dbg, nullptr, nullptr,
                                                        nullptr, dev_status, stream, dflash::sel::WalkArgs{});
}

extern "C" int dflash_select_verify(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                                    const dflash_bf16* Msel, const int32_t* target, int B, int L, int K, int r,
                                    int V, int32_t* path_tok, int32_t* path_slot, float* path_score,
                                    int32_t* accept_len, int32_t* next_token, int* dev_status, void* stream) {
  if (!target || !accept_len || !next_token) return DFLASH_ERR_INVALID_ARG;
  return dflash::sel::launch<dflash::sel::WALK_VITERBI>(topk_logp, topk_idx, E, Msel, B, L, K, r, V, path_tok,
                                                        path_slot, path_score, nullptr, target, accept_len,
                                                        next_token, dev_status, stream, dflash::sel::WalkArgs{});
}

extern "C" int dflash_path_walk(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                                const dflash_bf16* Msel, const int32_t* anchor, const float* uniforms,
                                float temperature, int B, int L, int K, int r, int V, int32_t* path_tok,
                                int32_t* path_slot, float* path_score, float* path_q, const int32_t* target,
                                int32_t* accept_len, int32_t* next_token, int* dev_status, void* stream) {
  using namespace dflash::sel;
  if (!anchor) return DFLASH_ERR_INVALID_ARG;
  if (target && (!accept_len || !next_token)) return DFLASH_ERR_INVALID_ARG;
  WalkArgs wa{anchor, uniforms, 0.f, path_q};
  if (uniforms == nullptr)
    return launch<WALK_GREEDY>(topk_logp, topk_idx, E, Msel, B, L, K, r, V, path_tok, path_slot, path_score, nullptr,
                               target, accept_len, next_token, dev_status, stream, wa);
  if (!(temperature > 0.f) || !(temperature < INFINITY)) return DFLASH_ERR_INVALID_ARG;
  wa.inv_t = 1.f / temperature;
  return launch<WALK_SAMPLE>(topk_logp, topk_idx, E, Msel, B, L, K, r, V, path_tok, path_slot, path_score, nullptr,
                             target, accept_len, next_token, dev_status, stream, wa);
}
