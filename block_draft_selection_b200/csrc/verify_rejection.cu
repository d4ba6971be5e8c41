// Rejection-sampling verification against the target's distributions.
//
// "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector",
// and "Inco AI's DFlash 2 lifts LLM decoding output 16-25%": a path drawn by
// sampling is verified by rejection sampling, which keeps the target's output
// distribution exactly.  Standard speculative sampling:
//   p_i = softmax(z_i / T) over the vocabulary (target logits z_i, row
//         b*(L+1)+i), q_i the distribution draft slot s_i was drawn from;
//   keep x_i while u_i * q_i(s_i) <= p_i(x_i); at the first rejection n emit
//   a draw from max(0, p_n - q_n) (q_n lives on the 16 candidates), after L
//   acceptances a draw from p_L; each draw by inverse CDF in vocabulary
//   order (the smallest token whose cumulative mass exceeds u * total).
//
// Two kernels:
//   1. row statistics: CTA (row, slice) reduces 8192 logits of one row to
//      (m, s) with c = log2(e) / T: m = c * max z (the slice's max, found
//      first), s = sum of exp2((z - max z) * c) (fp32 exponentials added in
//      pairs in fp32, the pair sums in fp64) -- also the slice's probability
//      mass once the row is merged;
//   2. one CTA of 1024 threads per block: merges its L+1 rows' statistics
//      (a warp per row: the max over the slices, then one fp64 rescale per
//      slice), tests the L drafts (one lane each), picks the residual's slice
//      from the slice masses (corrected at the 16 candidates), then scans
//      that slice's 8192 entries with a block-wide fp64 prefix sum: each
//      thread loads its 8 logits before any arithmetic and tests its range
//      against the 16 candidates once.  Every value that decides an outcome
//      here (p at a draft token, the entries of the scanned slice) is an
//      fp64 exponential.
#include <climits>

#include "common.cuh"

namespace dflash {
namespace rej {

constexpr int SPAN = 8192;          // logits per slice
constexpr int T1 = 256;             // threads of the row-statistics kernel
constexpr int EPT1 = SPAN / T1;     // 32 logits per thread
constexpr int T2 = 1024;            // threads of the per-block kernel
constexpr int EPT2 = SPAN / T2;     // 8 entries per thread in the final scan
constexpr int MAX_SLICES = 64;      // V <= 64 * 8192
constexpr int MAX_L = 31;           // L + 1 rows merged by L + 1 warps
constexpr int KC = 16;
constexpr unsigned FULL = 0xffffffffu;

struct Part {  // statistics of one slice of one row (16 bytes)
  double m;    // max of z*c over the slice (-inf: empty)
  double s;    // sum of exp2(z*c - m)
};

__global__ void __launch_bounds__(T1) row_stats_kernel(const float* __restrict__ z, int V, int S, double c, int vec,
                                                       Part* __restrict__ part) {
  pdl_wait();  // the logits may come from the kernel before this one
  pdl_trigger();
  const size_t row = blockIdx.x;
  const int split = blockIdx.y;
  const float* zr = z + row * V;
  const int v0 = split * SPAN;
  const int tid = threadIdx.x;
  float x[EPT1];
  if (vec) {
#pragma unroll
    for (int j = 0; j < EPT1 / 4; ++j) {
      const int v = v0 + (j * T1 + tid) * 4;
      float4 t = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (v < V) t = __ldg(reinterpret_cast<const float4*>(zr + v));  // V % 4 == 0: all four in range
      x[4 * j + 0] = t.x;
      x[4 * j + 1] = t.y;
      x[4 * j + 2] = t.z;
      x[4 * j + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < EPT1; ++j) {
      const int v = v0 + j * T1 + tid;
      x[j] = v < V ? __ldg(zr + v) : -INFINITY;
    }
  }
  // the slice's maximum first (fp32, exact), then every exponential against it
  __shared__ float wmax[T1 / 32];
  __shared__ double wsum[T1 / 32];
  const int warp = tid >> 5, lane = tid & 31;
  float xm = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPT1; ++j) xm = fmaxf(xm, x[j]);
#pragma unroll
  for (int off = 16; off; off >>= 1) xm = fmaxf(xm, __shfl_xor_sync(FULL, xm, off));
  if (lane == 0) wmax[warp] = xm;
  __syncthreads();
  xm = wmax[0];
#pragma unroll
  for (int w = 1; w < T1 / 32; ++w) xm = fmaxf(xm, wmax[w]);
  double s = 0.0;
  if (xm != -INFINITY) {
    // exp2((x - xm) * c) in fp32; neighbouring pairs added in fp32 (one
    // rounding, at most 2^-24 relative, below exp2f's own error), the pair
    // sums widened and added in fp64.  x - xm is exact wherever x >= xm / 2
    // (the terms that carry the sum) and otherwise off by at most 2^-24 of a
    // difference whose term is tiny; the product adds one rounding relative
    // to the exponent, i.e. |y| * 2^-24 * ln 2 relative to the term.
    const float cf = static_cast<float>(c);
#pragma unroll
    for (int j = 0; j < EPT1; j += 2)
      s += static_cast<double>(exp2f((x[j] - xm) * cf) + exp2f((x[j + 1] - xm) * cf));   // padding: 0
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(FULL, s, off);
  if (lane == 0) wsum[warp] = s;
  __syncthreads();
  if (tid == 0) {
    double sb = 0.0;
#pragma unroll
    for (int w = 0; w < T1 / 32; ++w) sb += wsum[w];
    Part p;
    p.m = static_cast<double>(xm) * c;   // c > 0: the max of z*c is at the max of z
    p.s = sb;
    part[row * S + split] = p;
  }
}

__global__ void __launch_bounds__(T2) reject_kernel(
    const float* __restrict__ z, int V, int S, double c, int vec, int L, const Part* __restrict__ part,
    const int32_t* __restrict__ draft, const int32_t* __restrict__ draft_slot, const int32_t* __restrict__ cand_idx,
    const float* __restrict__ draft_q, const float* __restrict__ u_accept, const float* __restrict__ u_resample,
    int32_t* __restrict__ accept_len, int32_t* __restrict__ next_token, int* status) {
  __shared__ double row_m[MAX_L + 1];
  __shared__ double row_s[MAX_L + 1];
  __shared__ double mass[MAX_SLICES];
  __shared__ Part parts_s[MAX_L + 1][MAX_SLICES];   // every row's slice statistics, read once
  __shared__ int cand_s[KC];
  __shared__ float q_s[KC];
  __shared__ double wsum[T2 / 32];
  __shared__ int sh_n, sh_slice, sh_pick, sh_before, sh_last;
  __shared__ double sh_excl, sh_target;
  __shared__ int pc_idx[MAX_L][KC];    // every position's candidates, their q and logits,
  __shared__ float pc_q[MAX_L][KC];    // read up front (the rejected position is not yet
  __shared__ float pc_z[MAX_L][KC];    // known, and these loads need not wait for it)

  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t row0 = static_cast<size_t>(b) * (L + 1);
  if (tid == 0) {
    sh_pick = INT_MAX;
    sh_before = -1;
    sh_last = -1;
  }
  // The drafts, their candidates and probabilities, the uniforms and the
  // target logits are read before the dependency wait, while the statistics
  // kernel runs: this kernel starts only once every statistics CTA has
  // triggered it, which each does after its own wait on the kernel before
  // it, so all of these are complete and visible here (without programmatic
  // launch the statistics kernel has simply finished).
  // warp 0, lane i < L: drafted position i's token, slot, q and target logit
  int dx = 0;
  double dq = 0.0, du = 0.0;
  float dz = 0.f;
  const float ures = warp == 0 ? u_resample[b] : 0.f;   // used in D
  if (warp == 0 && lane < L) {
    const size_t di = static_cast<size_t>(b) * L + lane;
    dx = draft[di];
    int sl = draft_slot[di];
    if (dx < 0 || dx >= V || sl < 0 || sl >= KC) {
      set_status(status, DFLASH_ERR_BAD_INDEX);
      dx = min(max(dx, 0), V - 1);
      sl = min(max(sl, 0), KC - 1);
    }
    dq = draft_q[di * KC + sl];
    du = u_accept[di];
    dz = z[(row0 + lane) * V + dx];
  }
  // threads 32 .. 32 + 16 L - 1: candidate k of position i
  if (tid >= 32 && tid < 32 + KC * L) {
    const int i = (tid - 32) / KC;
    const int k = (tid - 32) - i * KC;
    const size_t ci = (static_cast<size_t>(b) * L + i) * KC + k;
    int v = cand_idx[ci];
    float zv = 0.f;
    if (v < 0 || v >= V) {
      set_status(status, DFLASH_ERR_BAD_INDEX);
      v = -1;
    } else {
      zv = z[(row0 + i) * V + v];
    }
    pc_idx[i][k] = v;
    pc_q[i][k] = draft_q[ci];
    pc_z[i][k] = zv;
  }
  pdl_wait();   // the slice statistics
  pdl_trigger();

  // A. each row's max and sum from its slices (warp i -> row i; lane j holds
  // slices j and j + 32): the warp's max first, then one rescale per slice
  if (warp <= L) {
    Part p0{-INFINITY, 0.0}, p1{-INFINITY, 0.0};
    const Part* pr = part + (row0 + warp) * S;
    if (lane < S) p0 = pr[lane];
    if (lane + 32 < S) p1 = pr[lane + 32];
    if (lane < S) parts_s[warp][lane] = p0;
    if (lane + 32 < S) parts_s[warp][lane + 32] = p1;
    double m = fmax(p0.m, p1.m);
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmax(m, __shfl_xor_sync(FULL, m, off));
    double s = 0.0;
    if (m != -INFINITY) {
      if (p0.m != -INFINITY) s += p0.s * exp2(p0.m - m);
      if (p1.m != -INFINITY) s += p1.s * exp2(p1.m - m);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(FULL, s, off);
    if (lane == 0) {
      row_m[warp] = m;
      row_s[warp] = s;
    }
  }
  __syncthreads();

  // B. acceptance tests, lane i for drafted position i (values read above)
  if (warp == 0) {
    bool reject = false;
    if (lane < L) {
      const double p = exp2(static_cast<double>(dz) * c - row_m[lane]) / row_s[lane];
      reject = !(du * dq <= p);
    }
    const unsigned mask = __ballot_sync(FULL, reject);
    const int n = mask ? __ffs(mask) - 1 : L;
    if (lane == 0) {
      sh_n = n;
      accept_len[b] = n + 1;
    }
  }
  __syncthreads();
  const int n = sh_n;
  const size_t R = row0 + n;  // the row the next token is drawn from
  const double mx = row_m[n];
  const double inv_sR = 1.0 / row_s[n];   // one division; each probability below is a product
  const float* zr = z + R * V;

  // C. slice masses of p_R, minus q_n at the candidates (rejection only)
  if (tid < KC) {
    cand_s[tid] = n < L ? pc_idx[n][tid] : -1;
    q_s[tid] = n < L ? pc_q[n][tid] : 0.f;
  }
  for (int j = tid; j < S; j += T2) {
    const Part p = parts_s[n][j];
    mass[j] = p.m == -INFINITY ? 0.0 : exp2(p.m - mx) * p.s * inv_sR;
  }
  __syncthreads();
  if (tid < KC && cand_s[tid] >= 0) {
    const int v = cand_s[tid];
    const double pv = exp2(static_cast<double>(pc_z[n][tid]) * c - mx) * inv_sR;
    atomicAdd(&mass[v / SPAN], fmax(0.0, pv - static_cast<double>(q_s[tid])) - pv);
  }
  __syncthreads();

  // D. the slice the draw falls in (warp 0; two slices per lane, in order)
  if (warp == 0) {
    const int j0 = 2 * lane, j1 = 2 * lane + 1;
    const double m0 = j0 < S ? fmax(mass[j0], 0.0) : 0.0;
    const double m1 = j1 < S ? fmax(mass[j1], 0.0) : 0.0;
    double incl = m0 + m1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double t = __shfl_up_sync(FULL, incl, off);
      if (lane >= off) incl += t;
    }
    const double excl = incl - (m0 + m1);
    const double total = __shfl_sync(FULL, incl, 31);
    const double target = static_cast<double>(ures) * total;
    const unsigned over = __ballot_sync(FULL, incl > target);
    const unsigned pos = __ballot_sync(FULL, m0 > 0.0 || m1 > 0.0);
    if (lane == 0) sh_target = target;
    if (over) {
      if (lane == __ffs(over) - 1) {
        const bool first = excl + m0 > target;
        sh_slice = first ? j0 : j1;
        sh_excl = first ? excl : excl + m0;
      }
    } else {
      // u * total rounded up to total: the last slice with mass
      const int lp = pos ? 31 - __clz(pos) : 0;
      if (lane == lp) {
        const bool second = m1 > 0.0;
        sh_slice = second ? j1 : j0;
        sh_excl = second ? excl + m0 : excl;
      }
    }
  }
  __syncthreads();

  // E. inverse CDF inside the slice: block-wide prefix sum of the residual.
  // Each thread's 8 consecutive logits are loaded before any arithmetic (as
  // two 16-byte loads where the row allows it), and its range is tested
  // against the 16 candidates once.
  const int js = sh_slice;
  const double target = sh_target;
  const int v0 = js * SPAN + tid * EPT2;
  float zv[EPT2];
  if (vec) {
    // V % 4 == 0 and v0 % 8 == 0: a quad that starts inside the row ends inside it
    const float4 lo = v0 < V ? __ldg(reinterpret_cast<const float4*>(zr + v0)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 hi = v0 + 4 < V ? __ldg(reinterpret_cast<const float4*>(zr + v0 + 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    zv[0] = lo.x; zv[1] = lo.y; zv[2] = lo.z; zv[3] = lo.w;
    zv[4] = hi.x; zv[5] = hi.y; zv[6] = hi.z; zv[7] = hi.w;
  } else {
#pragma unroll
    for (int e = 0; e < EPT2; ++e) zv[e] = v0 + e < V ? __ldg(zr + v0 + e) : 0.f;
  }
  bool has_cand = false;
#pragma unroll
  for (int k = 0; k < KC; ++k) has_cand |= static_cast<unsigned>(cand_s[k] - v0) < static_cast<unsigned>(EPT2);
  double r[EPT2];
  double tsum = 0.0;
  int last_pos = -1;
#pragma unroll
  for (int e = 0; e < EPT2; ++e) {
    const int v = v0 + e;
    double rv = 0.0;
    if (v < V) {
      rv = exp2(static_cast<double>(zv[e]) * c - mx) * inv_sR;
      if (has_cand) {
        // which candidate (if any) is entry v: integer selects only, then
        // one fp64 correction (the candidates are distinct)
        int hit = -1;
#pragma unroll
        for (int k = 0; k < KC; ++k) hit = cand_s[k] == v ? k : hit;
        if (hit >= 0) rv = fmax(0.0, rv - static_cast<double>(q_s[hit]));
      }
    }
    r[e] = rv;
    tsum += rv;
    if (rv > 0.0) last_pos = v;
  }
  double incl = tsum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const double t = __shfl_up_sync(FULL, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    double w = wsum[lane];
    double wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double t = __shfl_up_sync(FULL, wi, off);
      if (lane >= off) wi += t;
    }
    wsum[lane] = wi - w;  // exclusive
  }
  __syncthreads();
  const double start = sh_excl + wsum[warp] + (incl - tsum);
  if (start <= target) {
    double run = start;
    int pick = -1;
#pragma unroll
    for (int e = 0; e < EPT2; ++e) {
      run += r[e];
      if (pick < 0 && run > target && r[e] > 0.0) pick = v0 + e;
    }
    if (pick >= 0) atomicMin(&sh_pick, pick);
    if (last_pos >= 0) atomicMax(&sh_before, last_pos);
  }
  if (last_pos >= 0) atomicMax(&sh_last, last_pos);
  __syncthreads();
  if (tid == 0) {
    // rounding fallbacks: the last entry with mass at or before the target,
    // else the last entry with mass in the slice
    int v = sh_pick != INT_MAX ? sh_pick : (sh_before >= 0 ? sh_before : sh_last);
    if (v < 0) v = min(js * SPAN, V - 1);
    next_token[b] = v;
  }
}

inline int slices(int V) { return (V + SPAN - 1) / SPAN; }

}  // namespace rej
}  // namespace dflash

extern "C" size_t dflash_verify_rejection_workspace(int B, int L, int V) {
  using namespace dflash::rej;
  if (B < 1 || L < 1 || V < 1) return 0;
  return static_cast<size_t>(B) * (L + 1) * slices(V) * sizeof(Part);
}

extern "C" int dflash_verify_rejection(const float* target_logits, float temperature, const int32_t* draft,
                                       const int32_t* draft_slot, const int32_t* cand_idx, const float* draft_q,
                                       const float* u_accept, const float* u_resample, int B, int L, int V,
                                       int32_t* accept_len, int32_t* next_token, void* ws, size_t ws_bytes,
                                       int* dev_status, void* stream) {
  using namespace dflash::rej;
  if (!target_logits || !draft || !draft_slot || !cand_idx || !draft_q || !u_accept || !u_resample ||
      !accept_len || !next_token)
    return DFLASH_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || L > MAX_L || V < 1 || V > MAX_SLICES * SPAN) return DFLASH_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !(temperature < INFINITY)) return DFLASH_ERR_INVALID_ARG;
  if (B > 0x7fffffff / (L + 1)) return DFLASH_ERR_INVALID_ARG;
  const size_t need = dflash_verify_rejection_workspace(B, L, V);
  if (!ws || ws_bytes < need) return DFLASH_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 15) return DFLASH_ERR_INVALID_ARG;
  const int S = slices(V);
  const double c = 1.4426950408889634 / static_cast<double>(temperature);  // log2(e) / T
  const int vec = (V % 4 == 0) && (reinterpret_cast<uintptr_t>(target_logits) % 16 == 0);
  const int rows = B * (L + 1);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  Part* part = static_cast<Part*>(ws);
  cudaError_t e = dflash::launch_kernel(row_stats_kernel, dim3(rows, S), dim3(T1), 0, st, target_logits, V, S, c,
                                        vec, part);
  if (e != cudaSuccess) return DFLASH_ERR_CUDA;
  e = dflash::launch_kernel(reject_kernel, dim3(B), dim3(T2), 0, st, target_logits, V, S, c, vec, L,
                            static_cast<const Part*>(part), draft, draft_slot, cand_idx, draft_q, u_accept,
                            u_resample, accept_len, next_token, dev_status);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
