// The pages' context-gated pair scorer and the walks over its scores.
//
// "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
// for the previous token a and a candidate b at position t,
//   S_t(a, b) = U_t(b) + < A(a) (.) H(h_t), B(b) >
// with compact e-dimensional token embeddings A, B and a context gate H.
// Here A(a) = Pa.emb(a), B(b) = Pb.emb(b) (Pab = [Pa; Pb], [2e, d]),
// H(h_t) = sigmoid(Pg.h_t) (Pg [e, d]) and U_t(b) the drafter's log-probability.
//
// A and B are functions of the token alone: dflash_ctx_table tabulates them
// once for the whole vocabulary, tab = Emb . Pab^T [V, 2e], and a cycle only
// reads the rows of its anchor and candidates.  dflash_ctx_gate computes
// gate = H . Pg^T [B L, e] (before the sigmoid).  Both are the library's
// tcgen05 GEMM.
//
// dflash_ctx_walk: one thread-block cluster of Q CTAs per block; CTA q scores
// tables t = q, q+Q, ... (table t: predecessor = the anchor for t = 0, else
// position t-1's candidates; successor = position t's candidates):
//   w[j][:] = A(pred_j) * sigmoid(gate_t)    (16 x e, shared memory)
//   S[j][k] = lp[t][k] + w[j] . B(c_tk)      (one thread per (j, k))
// written into the leader CTA's shared memory; the leader's warp 0 then walks
// them (max-sum from the anchor, greedy, or sampled; walk.cuh).
#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
#include "walk.cuh"

namespace dflash {
namespace ctx {

using namespace walk;

constexpr int THREADS = 256;
constexpr int KC = 16;
constexpr int MAX_CLUSTER = 8;
constexpr int MAX_E = 1024;

struct Layout {
  int ep;  // padded row length of the w / B buffers (floats)
  size_t s_off, tok_off, bp_off, ps_off, w_off, b_off, g_off, total;
};

__host__ __device__ inline Layout layout(int L, int e) {
  Layout o;
  o.ep = e + 4;
  size_t off = 0;
  o.s_off = off;
  off += static_cast<size_t>(L) * KC * KC * 4;
  o.tok_off = off;
  off += static_cast<size_t>(L + 1) * KC * 4;
  o.ps_off = off;
  off += static_cast<size_t>(L + 1) * 4;
  o.bp_off = off;
  off += static_cast<size_t>(L) * KC;
  off = (off + 15) & ~size_t(15);
  o.w_off = off;
  off += static_cast<size_t>(KC) * o.ep * 4;
  o.b_off = off;
  off += static_cast<size_t>(KC) * o.ep * 4;
  o.g_off = off;
  off += static_cast<size_t>(e) * 4;
  o.total = (off + 15) & ~size_t(15);
  return o;
}

template <int WALK>
__global__ void __launch_bounds__(THREADS) ctx_walk_kernel(
    const float* __restrict__ topk_logp, const int32_t* __restrict__ topk_idx, const float* __restrict__ tab,
    const float* __restrict__ gate, int L, int e, int V, int Q, WalkArgs wa, int32_t* __restrict__ path_tok,
    int32_t* __restrict__ path_slot, float* __restrict__ path_score, float* __restrict__ tables_dbg,
    const int32_t* __restrict__ target, int32_t* __restrict__ accept_len, int32_t* __restrict__ next_token,
    int* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  const Layout lo = layout(L, e);
  float* Ss = reinterpret_cast<float*>(smem + lo.s_off);
  int* toks = reinterpret_cast<int*>(smem + lo.tok_off);
  int* pslot = reinterpret_cast<int*>(smem + lo.ps_off);
  int8_t* bps = reinterpret_cast<int8_t*>(smem + lo.bp_off);
  float* Wb = reinterpret_cast<float*>(smem + lo.w_off);
  float* Bb = reinterpret_cast<float*>(smem + lo.b_off);
  float* gb = reinterpret_cast<float*>(smem + lo.g_off);

  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x / Q;
  const int q_rank = blockIdx.x - b * Q;
  const int tid = threadIdx.x;
  const size_t row0 = static_cast<size_t>(b) * L;
  const int e4 = e / 4;
  const size_t tw = 2 * static_cast<size_t>(e);   // floats per table row
  int pre_t = 0;
  float pre_u = 0.f;
  if (q_rank == 0 && tid < 32) {
    if (target != nullptr && tid <= L) pre_t = __ldg(target + static_cast<size_t>(b) * (L + 1) + tid);
    if (WALK == WALK_SAMPLE && tid < L) pre_u = __ldg(wa.uniforms + row0 + tid);
  }
  float* S_out = Ss;
  if (Q > 1) {
    S_out = cooperative_groups::this_cluster().map_shared_rank(Ss, 0);
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  }
  {
    // the walk's tokens: internal position 0 = the anchor (16 copies), then
    // the candidates of drafted positions 0..L-1 (every CTA: they pick the
    // table rows; the leader's copy also feeds the walk)
    for (int q = tid; q < (L + 1) * KC; q += THREADS) {
      int c;
      if (q < KC) {
        c = __ldg(wa.anchor + b);
      } else {
        c = __ldg(topk_idx + row0 * KC + (q - KC));
      }
      if (c < 0 || c >= V) {
        set_status(status, DFLASH_ERR_BAD_INDEX);
        c = 0;
      }
      toks[q] = c;
    }
  }
  if (Q > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");

  for (int t = q_rank; t < L; t += Q) {
    // gate of position t, predecessors' A rows (times the gate), successors' B rows
    for (int q = tid; q < e; q += THREADS) {
      const float x = __ldg(gate + (row0 + t) * e + q);
      gb[q] = 1.f / (1.f + expf(-x));
    }
    __syncthreads();
    for (int q = tid; q < KC * e4; q += THREADS) {
      const int j = q / e4;
      const int c4 = q - j * e4;
      // predecessor j: internal position t; successor j: internal position t + 1
      const size_t prow = static_cast<size_t>(toks[t * KC + j]);
      const size_t srow = static_cast<size_t>(toks[(t + 1) * KC + j]);
      const float4 a = __ldg(reinterpret_cast<const float4*>(tab + prow * tw) + c4);
      const float4 g = *reinterpret_cast<const float4*>(gb + 4 * c4);
      *reinterpret_cast<float4*>(Wb + j * lo.ep + 4 * c4) = make_float4(a.x * g.x, a.y * g.y, a.z * g.z, a.w * g.w);
      *reinterpret_cast<float4*>(Bb + j * lo.ep + 4 * c4) =
          __ldg(reinterpret_cast<const float4*>(tab + srow * tw + e) + c4);
    }
    __syncthreads();
    {
      const int j = tid >> 4;
      const int k = tid & 15;
      const float* wr = Wb + j * lo.ep;
      const float* br = Bb + k * lo.ep;
      float acc0 = 0.f, acc1 = 0.f;
      for (int q = 0; q < e; q += 8) {  // e % 8 == 0: two independent chains
        const float4 w0 = *reinterpret_cast<const float4*>(wr + q);
        const float4 b0 = *reinterpret_cast<const float4*>(br + q);
        const float4 w1 = *reinterpret_cast<const float4*>(wr + q + 4);
        const float4 b1 = *reinterpret_cast<const float4*>(br + q + 4);
        acc0 = fmaf(w0.x, b0.x, acc0);
        acc1 = fmaf(w1.x, b1.x, acc1);
        acc0 = fmaf(w0.y, b0.y, acc0);
        acc1 = fmaf(w1.y, b1.y, acc1);
        acc0 = fmaf(w0.z, b0.z, acc0);
        acc1 = fmaf(w1.z, b1.z, acc1);
        acc0 = fmaf(w0.w, b0.w, acc0);
        acc1 = fmaf(w1.w, b1.w, acc1);
      }
      const float sc = __ldg(topk_logp + (row0 + t) * KC + k) + (acc0 + acc1);
      S_out[(t * KC + j) * KC + k] = sc;
      if (tables_dbg) tables_dbg[((row0 + t) * KC + j) * KC + k] = sc;
    }
    __syncthreads();
  }

  if (Q > 1) {
    cooperative_groups::this_cluster().sync();  // every CTA's tables have landed
    if (q_rank != 0) return;
  } else {
    __syncthreads();
  }
  if (tid >= 32) return;
  if (WALK == WALK_VITERBI) {
    walk_maxsum(Ss, toks, L, 1, L, b, bps, pslot, pre_t, path_tok, path_slot, path_score, target != nullptr,
                accept_len, next_token);
  } else {
    walk_from_anchor<WALK>(Ss, toks, L, b, wa, pre_t, pre_u, path_tok, path_slot, path_score, target != nullptr,
                           accept_len, next_token);
  }
}

template <int WALK>
static int launch_walk(const float* topk_logp, const int32_t* topk_idx, const float* tab, const float* gate, int B,
                       int L, int e, int V, WalkArgs wa, int32_t* path_tok, int32_t* path_slot, float* path_score,
                       float* tables_dbg, const int32_t* target, int32_t* accept_len, int32_t* next_token,
                       int* dev_status, cudaStream_t st) {
  const Layout lo = layout(L, e);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(ctx_walk_kernel<WALK>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  });
  if (attr_err != cudaSuccess) return DFLASH_ERR_CUDA;
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int Q = 1;
  if (B * 2 < sms && L > 1) {
    Q = L < MAX_CLUSTER ? L : MAX_CLUSTER;
    while (Q > 1 && static_cast<long long>(B) * Q > sms) --Q;
  }
  const cudaError_t e2 = launch_kernel_cluster(ctx_walk_kernel<WALK>, dim3(B * Q), dim3(THREADS), lo.total, st, Q,
                                               topk_logp, topk_idx, tab, gate, L, e, V, Q, wa, path_tok, path_slot,
                                               path_score, tables_dbg, target, accept_len, next_token, dev_status);
  return e2 == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

}  // namespace ctx
}  // namespace dflash

extern "C" int dflash_ctx_table(const dflash_bf16* Emb, const dflash_bf16* Pab, int V, int d, int e, float* tab,
                                void* stream) {
  using namespace dflash::ctx;
  if (!Emb || !Pab || !tab) return DFLASH_ERR_INVALID_ARG;
  if (V < 1 || d < 8 || d % 8 != 0 || e < 16 || e > MAX_E || e % 8 != 0) return DFLASH_ERR_INVALID_ARG;
  return dflash_gemm_bf16(Emb, Pab, tab, V, 2 * e, d, stream);
}

extern "C" int dflash_ctx_gate(const dflash_bf16* H, const dflash_bf16* Pg, int M, int d, int e, float* gate,
                               void* stream) {
  using namespace dflash::ctx;
  if (!H || !Pg || !gate) return DFLASH_ERR_INVALID_ARG;
  if (M < 1 || d < 8 || d % 8 != 0 || e < 16 || e > MAX_E || e % 8 != 0) return DFLASH_ERR_INVALID_ARG;
  return dflash_gemm_bf16(H, Pg, gate, M, e, d, stream);
}

extern "C" int dflash_ctx_walk(const float* topk_logp, const int32_t* topk_idx, const int32_t* anchor,
                               const float* tab, const float* gate, int B, int L, int K, int e, int V, int walk,
                               const float* uniforms, float temperature, int32_t* path_tok, int32_t* path_slot,
                               float* path_score, float* path_q, float* tables_dbg, const int32_t* target,
                               int32_t* accept_len, int32_t* next_token, int* dev_status, void* stream) {
  using namespace dflash::ctx;
  if (!topk_logp || !topk_idx || !anchor || !tab || !gate || !path_tok) return DFLASH_ERR_INVALID_ARG;
  if (K != KC || B < 1 || L < 1 || L > 16 || V < 1 || e < 16 || e > MAX_E || e % 8 != 0)
    return DFLASH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(tab) | reinterpret_cast<uintptr_t>(gate)) & 15) return DFLASH_ERR_INVALID_ARG;
  if (target && (!accept_len || !next_token)) return DFLASH_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  WalkArgs wa{anchor, uniforms, 0.f, path_q};
  switch (walk) {
    case 0:
      return launch_walk<WALK_VITERBI>(topk_logp, topk_idx, tab, gate, B, L, e, V, wa, path_tok, path_slot,
                                       path_score, tables_dbg, target, accept_len, next_token, dev_status, st);
    case 1:
      return launch_walk<WALK_GREEDY>(topk_logp, topk_idx, tab, gate, B, L, e, V, wa, path_tok, path_slot,
                                      path_score, tables_dbg, target, accept_len, next_token, dev_status, st);
    case 2:
      if (!uniforms || !(temperature > 0.f) || !(temperature < INFINITY)) return DFLASH_ERR_INVALID_ARG;
      wa.inv_t = 1.f / temperature;
      return launch_walk<WALK_SAMPLE>(topk_logp, topk_idx, tab, gate, B, L, e, V, wa, path_tok, path_slot,
                                      path_score, tables_dbg, target, accept_len, next_token, dev_status, st);
    default:
      return DFLASH_ERR_INVALID_ARG;
  }
}
