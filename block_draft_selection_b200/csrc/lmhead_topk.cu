// LM head + log-softmax + top-16, fused: the logits live only in TMEM and
// registers, never in HBM.
//
// What is computed ("DFlash 2: Keep Drafting Parallel", section "the right
// token is already in the candidates", Table 1: keep each drafted position's
// 16 best candidates out of the full vocabulary):
//   z[m,v] = H[m,:] . W[v,:],  lse[m] = log sum_v exp z[m,v],
//   top-16 of z[m,:] (value desc, index asc), logp = z - lse.
//
// Kernel 1 (lmhead_kernel) is a persistent, warp-specialised tcgen05 GEMM:
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles of W and H into
//               a ring of shared-memory stages (mbarrier transaction counts)
//   warp 1      MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32) into
//               a double-buffered TMEM accumulator; owns the TMEM allocation
//   warps 2..5  epilogue: tcgen05.ld the accumulator, keep an online
//               (max, sum exp) and a register-resident sorted top-16 per row,
//               write one partial record per (row, slot)
// Two tile orientations:
//   SWAP  (M <= 128, weight streaming): the MMA's M side is 128 vocabulary
//         rows of W, its N side the M tokens padded to 16.  Each CTA owns one
//         contiguous, balanced vocabulary range (16-row granularity; a ragged
//         last tile is fetched as 16-row boxes so no byte of W is read twice).
//         The epilogue transposes the tile through shared memory so threads
//         own tokens.  One partial per (row, CTA).
//   LARGE (M > 128, tensor bound): the MMA's M side is 128 token rows, its N
//         side 256 vocabulary columns; TMEM lane = token row, so each thread
//         scans its row directly.  Tiles are visited vocabulary-major so the
//         CTAs working at one time share W tiles through L2.  One partial per
//         (row, vocabulary tile).
// Kernel 2 (merge_kernel) folds a row's partials: one warp per row.
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "common.cuh"

namespace dflash {
namespace lm {

constexpr int BK = 64;                  // bf16 per K stage = one 128-byte swizzle row
constexpr int UMMA_K = 16;              // K per tcgen05.mma kind::f16
constexpr int A_ROWS = 128;             // MMA M
constexpr int A_STAGE_BYTES = A_ROWS * BK * 2;
constexpr int LARGE_N = 256;            // MMA N in LARGE mode
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int SMEM_BUDGET = 224 * 1024;

enum { MODE_SWAP = 0, MODE_LARGE = 1 };
// LARGE-orientation tile schedules:
//  STRIDED  tile t = cta + k * grid in vocabulary-major order: the CTAs running
//           at one time cover a narrow vocabulary window (W tiles are shared
//           through L2); each tile starts a fresh candidate list.
//  RUNS     CTA c owns m-tile (c % m_tiles) over one contiguous vocabulary range
//           (range c / m_tiles of nr); the CTAs owning one range walk it in
//           lockstep (W shared through L2) and each keeps its candidate list
//           across the whole range, so few values reach the insertion code.
enum { SCHED_STRIDED = 0, SCHED_RUNS = 1 };

struct Params {
  int M, V, d;
  int num_kc;        // K stages per tile = ceil(d / 64)
  int stages;        // shared-memory ring depth
  int n_mma;         // MMA N
  int tmem_cols;     // allocated TMEM columns (power of two >= 32)
  int buf_cols;      // TMEM columns per accumulator buffer
  int b_stage_bytes; // shared bytes of one B stage
  int b_tx_bytes;    // TMA bytes landing in one B stage
  // SWAP
  int units;         // ceil(V / 16)
  int g;             // epilogue threads per token
  int t_stride;      // floats per token row of the transpose buffer
  int t_bytes;
  // LARGE
  int m_tiles, v_tiles;
  int sched;         // SCHED_STRIDED or SCHED_RUNS
  int nr;            // SCHED_RUNS: vocabulary ranges per m-tile
  // outputs
  Partial* part;     // [M][P]
  int P;
  float* z_dbg;      // optional raw logits [M][V]
  int* status;
  unsigned long long timeout_ns;
};

struct SmemLayout {
  uint32_t a, b, t, bars, misc, total;
};

__host__ __device__ inline SmemLayout smem_layout(const Params& p) {
  SmemLayout s;
  s.a = 0;
  s.b = s.a + p.stages * A_STAGE_BYTES;
  s.t = s.b + p.stages * p.b_stage_bytes;
  s.bars = s.t + p.t_bytes;
  s.misc = s.bars + (2 * p.stages + 5) * 8;
  s.total = s.misc + 16;
  return s;
}

// ------------------------------------------------------------ tile walks ---

// SWAP: this CTA's balanced vocabulary range [r0, r1), a multiple of 16 rows.
__device__ __forceinline__ void swap_range(const Params& p, int& r0, int& r1) {
  const long long G = gridDim.x;
  const long long c = blockIdx.x;
  r0 = static_cast<int>((c * p.units) / G) * 16;
  r1 = static_cast<int>(((c + 1) * p.units) / G) * 16;
}

// LARGE: the k-th tile of this CTA; false past the end.  `slot` names the
// partial record the tile's run writes; first/last mark the run's ends.
__device__ __forceinline__ bool large_tile(const Params& p, int k, int& mt, int& vt, int& slot, bool& first,
                                           bool& last) {
  if (p.sched == SCHED_RUNS) {
    const int c = blockIdx.x;
    mt = c % p.m_tiles;
    const int r = c / p.m_tiles;
    const int lo = static_cast<int>(static_cast<long long>(r) * p.v_tiles / p.nr);
    const int hi = static_cast<int>(static_cast<long long>(r + 1) * p.v_tiles / p.nr);
    vt = lo + k;
    if (vt >= hi) return false;
    slot = r;
    first = k == 0;
    last = vt == hi - 1;
    return true;
  }
  const long long t = blockIdx.x + static_cast<long long>(k) * gridDim.x;
  if (t >= static_cast<long long>(p.m_tiles) * p.v_tiles) return false;
  vt = static_cast<int>(t / p.m_tiles);
  mt = static_cast<int>(t - static_cast<long long>(vt) * p.m_tiles);
  slot = vt;
  first = last = true;
  return true;
}

// ------------------------------------------------------------ kernel -------

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    lmhead_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a16,
                  const __grid_constant__ CUtensorMap tm_b, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemLayout L = smem_layout(p);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + L.bars;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (p.stages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * p.stages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * p.stages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * p.stages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  volatile int* epi_ok = reinterpret_cast<volatile int*>(smem + L.misc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), EPI_THREADS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *epi_ok = 1;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_a16);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up above overlaps the previous kernel; global memory only from here.
  pdl_wait();
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;

  int r0 = 0, r1 = 0;
  if (MODE == MODE_SWAP) swap_range(p, r0, r1);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      if (MODE == MODE_SWAP) {
        for (int t0 = r0; ok && t0 < r1; t0 += A_ROWS) {
          const int rows = min(A_ROWS, r1 - t0);
          for (int kc = 0; kc < p.num_kc; ++kc) {
            if (!mbar_wait(empty_bar(s), ph ^ 1u, deadline, abort_flag, p.status)) {
              ok = false;
              break;
            }
            const uint32_t fb = full_bar(s);
            mbar_arrive_expect_tx(fb, static_cast<uint32_t>(rows * BK * 2 + p.b_tx_bytes));
            const uint32_t a_dst = sbase + L.a + s * A_STAGE_BYTES;
            if (rows == A_ROWS) {
              tma_load_2d_hint(a_dst, &tm_a, fb, kc * BK, t0, pol_stream);
            } else {
              for (int j = 0; j < rows / 16; ++j)
                tma_load_2d_hint(a_dst + j * 16 * BK * 2, &tm_a16, fb, kc * BK, t0 + 16 * j, pol_stream);
            }
            tma_load_2d_hint(sbase + L.b + s * p.b_stage_bytes, &tm_b, fb, kc * BK, 0, pol_keep);
            issued_mask |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
            if (++s == p.stages) { s = 0; ph ^= 1u; }
          }
        }
      } else {
        int mt, vt, slot;
        bool first, last;
        for (int k = 0; ok && large_tile(p, k, mt, vt, slot, first, last); ++k) {
          for (int kc = 0; kc < p.num_kc; ++kc) {
            if (!mbar_wait(empty_bar(s), ph ^ 1u, deadline, abort_flag, p.status)) {
              ok = false;
              break;
            }
            const uint32_t fb = full_bar(s);
            mbar_arrive_expect_tx(fb, static_cast<uint32_t>(A_STAGE_BYTES + p.b_tx_bytes));
            tma_load_2d_hint(sbase + L.a + s * A_STAGE_BYTES, &tm_a, fb, kc * BK, mt * A_ROWS, pol_keep);
            // W tiles are shared by the m-tiles running at the same time: default L2 policy.
            tma_load_2d(sbase + L.b + s * p.b_stage_bytes, &tm_b, fb, kc * BK, vt * LARGE_N);
            issued_mask |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
            if (++s == p.stages) { s = 0; ph ^= 1u; }
          }
        }
      }
      if (!ok) {
        // Do not leave with copies in flight: wait (bounded) for the last
        // load issued into every stage to land.
        const uint64_t dl = globaltimer_ns() + 50000000ull;
        for (int q = 0; q < p.stages; ++q) {
          if (!(issued_mask >> q & 1u)) continue;
          const uint32_t par = (issued_par >> q) & 1u;
          while (!mbar_try_wait(full_bar(q), par) && globaltimer_ns() < dl) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(A_ROWS, p.n_mma);
      int s = 0;
      uint32_t ph = 0;
      int tb = 0;
      uint32_t tph = 0;
      bool ok = true;
      auto do_tile = [&]() -> bool {
        if (!mbar_wait(tempty_bar(tb), tph ^ 1u, deadline, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * p.buf_cols);
        for (int kc = 0; kc < p.num_kc; ++kc) {
          if (!mbar_wait(full_bar(s), ph, deadline, abort_flag, p.status)) return false;
          tc_fence_after();
          const uint64_t adesc = umma_desc_sw128(sbase + L.a + s * A_STAGE_BYTES);
          const uint64_t bdesc = umma_desc_sw128(sbase + L.b + s * p.b_stage_bytes);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            // advance the start address by k * 32 bytes (encoded >> 4)
            umma_bf16(d_tmem, adesc + 2ull * k, bdesc + 2ull * k, idesc, (kc | k) != 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
          if (++s == p.stages) { s = 0; ph ^= 1u; }
        }
        umma_commit(tfull_bar(tb));
        if (++tb == 2) { tb = 0; tph ^= 1u; }
        return true;
      };
      if (MODE == MODE_SWAP) {
        for (int t0 = r0; ok && t0 < r1; t0 += A_ROWS) ok = do_tile();
      } else {
        int mt, vt, slot;
        bool first, last;
        for (int k = 0; ok && large_tile(p, k, mt, vt, slot, first, last); ++k) ok = do_tile();
      }
      // Every MMA this thread issued has completed before TMEM is released.
      umma_commit(drain_bar);
      const uint64_t dl = globaltimer_ns() + 50000000ull;
      while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() < dl) {
      }
    }
  } else {
    // ------------------------------------------------------ epilogue ------
    const int e = threadIdx.x - 64;           // 0..127
    const int quarter = warp & 3;             // TMEM lanes this warp may access
    const int trow = quarter * 32 + lane;     // accumulator row held by this thread
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    TopState st;
    st.reset();
    int tb = 0;
    uint32_t tph = 0;

    if (MODE == MODE_SWAP) {
      float* T = reinterpret_cast<float*>(smem + L.t);
      const int g = p.g;
      const int n = e / g;
      const int sub = e - n * g;
      const bool active = n < p.M;
      const int ncols = (p.M + 15) & ~15;
      for (int t0 = r0; t0 < r1; t0 += A_ROWS) {
        const int rows = min(A_ROWS, r1 - t0);
        if (e == 0) *epi_ok = mbar_wait(tfull_bar(tb), tph, deadline, abort_flag, p.status) ? 1 : 0;
        named_barrier_sync(1, EPI_THREADS);
        if (!*epi_ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + static_cast<uint32_t>(tb * p.buf_cols) + lane_off;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float x[16];
          tmem_ld16(taddr + c0, x);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (c0 + jj < p.M) T[(c0 + jj) * p.t_stride + trow] = x[jj];
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(tb));
        if (++tb == 2) { tb = 0; tph ^= 1u; }
        named_barrier_sync(1, EPI_THREADS);
        if (active) {
          const float* Tn = T + n * p.t_stride;
          const int vend = min(rows, p.V - t0);
          for (int l = sub; l < vend; l += g) {
            const float x = Tn[l];
            const int v = t0 + l;
            if (p.z_dbg) p.z_dbg[static_cast<size_t>(n) * p.V + v] = x;
            if (x > st.m) {
              st.s = st.s * __expf(st.m - x) + 1.f;
              st.m = x;
            } else {
              st.s += __expf(x - st.m);
            }
            st.insert(x, v);
          }
        }
      }
      // Fold the g lists of each token (g adjacent lanes) into one.
      for (int off = 1; off < g; off <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, st.m, off);
        const float s2 = __shfl_xor_sync(0xffffffffu, st.s, off);
        st.merge_lse(m2, s2);
      }
      float ov[KTOP];
      int oi[KTOP];
#pragma unroll
      for (int r = 0; r < KTOP; ++r) {
        float bv = st.v[0];
        int bi = st.i[0];
        for (int off = 1; off < g; off <<= 1) {
          const float v2 = __shfl_xor_sync(0xffffffffu, bv, off);
          const int i2 = __shfl_xor_sync(0xffffffffu, bi, off);
          if (better(v2, i2, bv, bi)) {
            bv = v2;
            bi = i2;
          }
        }
        if (st.i[0] == bi && st.v[0] == bv) st.pop_head();
        ov[r] = bv;
        oi[r] = bi;
      }
      if (active && sub == 0) store_partial(p.part + static_cast<size_t>(n) * p.P + blockIdx.x, st.m, st.s, ov, oi);
    } else {
      int mt, vt, slot;
      bool first, last;
      for (int k = 0; large_tile(p, k, mt, vt, slot, first, last); ++k) {
        int ok = 0;
        if (lane == 0) ok = mbar_wait(tfull_bar(tb), tph, deadline, abort_flag, p.status) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        if (first) st.reset();
        const int row = mt * A_ROWS + trow;
        const int v0 = vt * LARGE_N;
        const uint32_t taddr = tmem_base + static_cast<uint32_t>(tb * p.buf_cols) + lane_off;
        for (int c0 = 0; c0 < LARGE_N && v0 + c0 < p.V; c0 += 16) {
          float x[16];
          tmem_ld16(taddr + c0, x);
          tmem_ld_wait();
          const int nvalid = min(16, p.V - (v0 + c0));
          float cmax = -INFINITY;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (jj < nvalid) cmax = fmaxf(cmax, x[jj]);
          if (cmax > st.m) {
            st.s *= __expf(st.m - cmax);
            st.m = cmax;
          }
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (jj < nvalid) st.s += __expf(x[jj] - st.m);
          // Candidates of this chunk that can enter the list; each lane then
          // inserts only its own, so the warp loops max_lane(count) times.
          uint32_t pend = 0;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (jj < nvalid && x[jj] >= st.v[KTOP - 1]) pend |= 1u << jj;
          while (__any_sync(0xffffffffu, pend != 0)) {
            if (pend) {
              const int jj = __ffs(pend) - 1;
              pend &= pend - 1;
              float xv = x[0];
#pragma unroll
              for (int q = 1; q < 16; ++q) xv = jj == q ? x[q] : xv;
              st.insert(xv, v0 + c0 + jj);
            }
          }
          if (p.z_dbg && row < p.M) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              if (jj < nvalid) p.z_dbg[static_cast<size_t>(row) * p.V + v0 + c0 + jj] = x[jj];
          }
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(tb));
        if (++tb == 2) { tb = 0; tph ^= 1u; }
        if (last && row < p.M) store_partial(p.part + static_cast<size_t>(row) * p.P + slot, st.m, st.s, st.v, st.i);
      }
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// One warp per row: fold P partial records into the final top-16 and lse.
__global__ void __launch_bounds__(128) merge_kernel(const Partial* __restrict__ part, int M, int P,
                                                    float* __restrict__ topk_logp,
                                                    int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (row >= M) return;
  TopState st;
  st.reset();
  const Partial* base = part + static_cast<size_t>(row) * P;
  // Records are loaded one ahead so the next load overlaps this record's work.
  PartialRegs cur, nxt;
  if (lane < P) cur.load(base + lane);
  for (int q = lane; q < P; q += 32) {
    if (q + 32 < P) nxt.load(base + q + 32);
    st.merge_lse(cur.m(), cur.s());
    float rv[KTOP];
    int ri[KTOP];
    cur.lists(rv, ri);
    st.insert_sorted(rv, ri);
    cur = nxt;
  }
  for (int off = 1; off < 32; off <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, st.m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, st.s, off);
    st.merge_lse(m2, s2);
  }
  const float row_lse = st.m + logf(st.s);
  float my_v = 0.f;
  int my_i = 0;
#pragma unroll
  for (int r = 0; r < KTOP; ++r) {
    float bv = st.v[0];
    int bi = st.i[0];
    for (int off = 1; off < 32; off <<= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, bv, off);
      const int i2 = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(v2, i2, bv, bi)) {
        bv = v2;
        bi = i2;
      }
    }
    if (st.i[0] == bi && st.v[0] == bv) st.pop_head();
    if (lane == r) {
      my_v = bv;
      my_i = bi;
    }
  }
  if (lane < KTOP) {
    topk_logp[static_cast<size_t>(row) * KTOP + lane] = my_v - row_lse;
    topk_idx[static_cast<size_t>(row) * KTOP + lane] = my_i;
  }
  if (lane == 0 && lse != nullptr) lse[row] = row_lse;
}

// ------------------------------------------------------------ host side ----

static int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

static unsigned long long timeout_ns_from_env() {
  static unsigned long long v = [] {
    const char* e = std::getenv("DFLASH_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms <= 0) ms = 2000;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return v;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// 2-D bf16 tensor [rows, cols] row-major, box [box_rows, 64], 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct Plan {
  int mode;
  int grid;
  Params p;
  size_t smem;
};

static bool make_plan(int M, int V, int d, int sms, Plan& pl) {
  if (M < 1 || V < 16 || d < 8 || d % 8 != 0 || sms < 1) return false;
  Params& p = pl.p;
  p = Params{};
  p.M = M;
  p.V = V;
  p.d = d;
  p.num_kc = (d + BK - 1) / BK;
  if (M <= 128) {
    pl.mode = MODE_SWAP;
    p.n_mma = (M + 15) & ~15;
    p.buf_cols = p.n_mma;
    int cols = 32;
    while (cols < 2 * p.n_mma) cols <<= 1;
    p.tmem_cols = cols;
    p.b_stage_bytes = p.n_mma * BK * 2;
    p.b_tx_bytes = p.b_stage_bytes;
    p.units = (V + 15) / 16;
    int g = 32;
    while (g > 1 && g * M > EPI_THREADS) g >>= 1;
    p.g = g;
    p.t_stride = 128 + g;
    p.t_bytes = ((M * p.t_stride * 4) + 1023) & ~1023;
    pl.grid = p.units < sms ? p.units : sms;
    p.P = pl.grid;
    const int fixed = p.t_bytes + 1024 + 512;
    int stages = (SMEM_BUDGET - fixed) / (A_STAGE_BYTES + p.b_stage_bytes);
    if (stages > 16) stages = 16;
    if (stages < 2) return false;
    p.stages = stages;
  } else {
    pl.mode = MODE_LARGE;
    p.n_mma = LARGE_N;
    p.buf_cols = LARGE_N;
    p.tmem_cols = 512;
    p.b_stage_bytes = LARGE_N * BK * 2;
    p.b_tx_bytes = p.b_stage_bytes;
    p.g = 1;
    p.t_stride = 0;
    p.t_bytes = 0;
    p.m_tiles = (M + A_ROWS - 1) / A_ROWS;
    p.v_tiles = (V + LARGE_N - 1) / LARGE_N;
    const long long tiles = static_cast<long long>(p.m_tiles) * p.v_tiles;
    const int g_str = static_cast<int>(tiles < sms ? tiles : sms);
    const long long t_str = (tiles + g_str - 1) / g_str;           // tiles on the busiest CTA
    int nr = sms / p.m_tiles;
    if (nr > p.v_tiles) nr = p.v_tiles;
    const long long t_run = nr >= 1 ? (p.v_tiles + nr - 1) / nr : (1ll << 40);
    if (t_run <= t_str) {
      p.sched = SCHED_RUNS;
      p.nr = nr;
      pl.grid = nr * p.m_tiles;
      p.P = nr;
    } else {
      p.sched = SCHED_STRIDED;
      p.nr = 0;
      pl.grid = g_str;
      p.P = p.v_tiles;
    }
    p.stages = 4;
  }
  pl.smem = smem_layout(p).total + 1024;
  return true;
}

static size_t part_bytes(const Plan& pl) {
  return static_cast<size_t>(pl.p.M) * pl.p.P * sizeof(Partial);
}

static int launch(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, float* topk_logp,
                  int32_t* topk_idx, float* lse, float* z_dbg, void* ws, size_t ws_bytes, int* dev_status,
                  void* stream) {
  if (!H || !W || !ws) return DFLASH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(H) & 15) || (reinterpret_cast<uintptr_t>(W) & 15) ||
      (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_ERR_INVALID_ARG;
  Plan pl;
  if (!make_plan(M, V, d, num_sms_current(), pl)) return DFLASH_ERR_INVALID_ARG;
  if (ws_bytes < part_bytes(pl)) return DFLASH_ERR_WORKSPACE;
  Params& p = pl.p;
  p.part = static_cast<Partial*>(ws);
  p.z_dbg = z_dbg;
  p.status = dev_status;
  p.timeout_ns = timeout_ns_from_env();

  CUtensorMap ta, ta16, tb;
  bool ok;
  if (pl.mode == MODE_SWAP) {
    ok = make_map(&ta, W, V, d, A_ROWS) && make_map(&ta16, W, V, d, 16) && make_map(&tb, H, M, d, p.n_mma);
  } else {
    ok = make_map(&ta, H, M, d, A_ROWS) && make_map(&tb, W, V, d, LARGE_N);
    ta16 = ta;
  }
  if (!ok) return DFLASH_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  static std::once_flag once[2];
  static cudaError_t attr_err[2] = {cudaSuccess, cudaSuccess};
  if (pl.mode == MODE_SWAP) {
    std::call_once(once[0], [] {
      attr_err[0] = cudaFuncSetAttribute(lmhead_kernel<MODE_SWAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BUDGET + 2048);
    });
    if (attr_err[0] != cudaSuccess) return DFLASH_ERR_CUDA;
    if (launch_kernel(lmhead_kernel<MODE_SWAP>, dim3(pl.grid), dim3(NUM_THREADS), pl.smem, st, ta, ta16, tb, p) !=
        cudaSuccess)
      return DFLASH_ERR_CUDA;
  } else {
    std::call_once(once[1], [] {
      attr_err[1] = cudaFuncSetAttribute(lmhead_kernel<MODE_LARGE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BUDGET + 2048);
    });
    if (attr_err[1] != cudaSuccess) return DFLASH_ERR_CUDA;
    if (launch_kernel(lmhead_kernel<MODE_LARGE>, dim3(pl.grid), dim3(NUM_THREADS), pl.smem, st, ta, ta16, tb, p) !=
        cudaSuccess)
      return DFLASH_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
  if (z_dbg == nullptr) {
    const int rows_per_cta = 4;
    if (launch_kernel(merge_kernel, dim3((M + rows_per_cta - 1) / rows_per_cta), dim3(32 * rows_per_cta), 0, st,
                      static_cast<const Partial*>(p.part), M, p.P, topk_logp, topk_idx, lse) != cudaSuccess)
      return DFLASH_ERR_CUDA;
  }
  return DFLASH_OK;
}

}  // namespace lm
}  // namespace dflash

extern "C" size_t dflash_lmhead_topk_workspace(int M, int V, int d) {
  dflash::lm::Plan pl;
  if (!dflash::lm::make_plan(M, V, d, dflash::lm::num_sms_current(), pl)) return 0;
  return dflash::lm::part_bytes(pl);
}

extern "C" int dflash_lmhead_topk(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, int K,
                                  float* topk_logp, int32_t* topk_idx, float* lse, void* ws, size_t ws_bytes,
                                  int* dev_status, void* stream) {
  if (K != dflash::KTOP || !topk_logp || !topk_idx) return DFLASH_ERR_INVALID_ARG;
  return dflash::lm::launch(H, W, M, V, d, topk_logp, topk_idx, lse, nullptr, ws, ws_bytes, dev_status, stream);
}

extern "C" int dflash_lmhead_logits_debug(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d,
                                          float* z, void* ws, size_t ws_bytes, int* dev_status, void* stream) {
  if (!z) return DFLASH_ERR_INVALID_ARG;
  return dflash::lm::launch(H, W, M, V, d, nullptr, nullptr, nullptr, z, ws, ws_bytes, dev_status, stream);
}

// ---------------------------------------------------------------------------
// No-allocation variant of dflash_lmhead_topk.
//
// Some callers cannot hand this library a device workspace: code running
// inside a custom allocator's own callbacks, engines whose memory pool is
// fully reserved up front, and hosts that forbid cudaMalloc after start-up
// (for example while other work is being captured or replayed).  For them,
// the per-row partial records live in the file-scope array below instead of
// a caller buffer.  The array is part of the library image: every GPU that
// loads libdflash.so holds DFLASH_STATIC_SCRATCH_BYTES of it until the
// process exits.
//
// Host code cannot use `g_static_scratch` as a pointer (its host-side name is
// only a stand-in for the device symbol), so the device address is looked up
// with cudaGetSymbolAddress once per device, with that device current, on the
// first call made while it is current.  That first call on a device should
// therefore happen before any stream capture begins.
//
// Every call shares the one array: calls that can overlap on the GPU (other
// streams, other host threads on the same device) race on it and must be
// serialised by the caller.  Nothing in it needs clearing between calls:
// every record the merge step reads is written earlier in the same call.
// ---------------------------------------------------------------------------

static __device__ __align__(256) unsigned char g_static_scratch[DFLASH_STATIC_SCRATCH_BYTES];

namespace dflash {
namespace lm {

constexpr int kMaxDevices = 64;
static std::mutex g_static_mu;
static void* g_static_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once).
static int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DFLASH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return DFLASH_ERR_CUDA;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return DFLASH_OK;
}

}  // namespace lm
}  // namespace dflash

extern "C" int dflash_lmhead_topk_static(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, int K,
                                         float* topk_logp, int32_t* topk_idx, float* lse, int* dev_status,
                                         void* stream) {
  if (K != dflash::KTOP || !topk_logp || !topk_idx || !H || !W) return DFLASH_ERR_INVALID_ARG;
  const size_t need = dflash_lmhead_topk_workspace(M, V, d);
  if (need == 0) return DFLASH_ERR_INVALID_ARG;
  if (need > static_cast<size_t>(DFLASH_STATIC_SCRATCH_BYTES)) return DFLASH_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int rc = dflash::lm::static_scratch(&scratch);
  if (rc != DFLASH_OK) return rc;
  return dflash::lm::launch(H, W, M, V, d, topk_logp, topk_idx, lse, nullptr, scratch,
                            static_cast<size_t>(DFLASH_STATIC_SCRATCH_BYTES), dev_status, stream);
}
