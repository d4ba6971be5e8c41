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
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles of H and W into
//               a ring of shared-memory stages (mbarrier transaction counts)
//   warp 1      MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32) into
//               a double-buffered TMEM accumulator; owns the TMEM allocation
//   warps 2..9  epilogue: TMEM lane = token row; two warps share each lane
//               quarter and split the tile's vocabulary columns; each thread
//               keeps an online (max, sum exp) and a register-resident sorted
//               top-16 and writes one partial record per (row, slot, half)
// The MMA's M side is always token rows and its N side up to 256 vocabulary
// rows of W: a tcgen05.mma of M = 128 costs about the same time for any N up
// to 256, so W goes on the N side where each instruction consumes 256 rows.
//   STREAM (M <= 128, weight streaming): one token tile (the A box holds the
//          M rows rounded up to 16; the MMA's other rows are never read back).
//          Each CTA owns one contiguous, balanced vocabulary range at 16-row
//          granularity; a ragged last tile is fetched as 16-row boxes and
//          multiplied with a narrower N, so no byte of W is read twice.
//   LARGE  (M > 128, tensor bound): token tiles of 128 rows, or 256 rows on a
//          cluster of two CTAs sharing one tcgen05.mma.cta_group::2 ("pair":
//          each CTA stages half of A and half of B, the leader issues the MMA
//          and each CTA's TMEM receives its 128 rows of D).  Tiles are either
//          vocabulary-strided (W shared through L2 across concurrent token
//          tiles) or long runs of one token tile over a vocabulary range.
// No load uses cluster multicast: every CTA fetches its own tiles.
// Kernel 2 (merge_kernel_rank) merges a row's partial records: one CTA per
// row picks the top-16 by a threshold and a parallel rank count.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace dflash {
namespace lm {

constexpr int BK = 64;                  // bf16 per K stage = one 128-byte swizzle row
constexpr int UMMA_K = 16;              // K per tcgen05.mma kind::f16
constexpr int A_ROWS = 128;             // token rows per CTA and MMA M of one CTA
constexpr int TILE_N = 256;             // vocabulary rows per tile (MMA N)
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int NUM_THREADS = 64 + EPI_THREADS;
constexpr int SMEM_BUDGET = 224 * 1024;
constexpr int MMA_A_SPAN = A_ROWS * BK * 2;  // shared bytes one MMA reads from an A stage

enum { MODE_STREAM = 0, MODE_LARGE = 1 };
// LARGE-orientation tile schedules (over work units = CTAs, or CTA pairs):
//  BLOCKS   the (token tile, block of R consecutive vocabulary tiles) jobs,
//           ordered block-major, go to units round-robin: the units running
//           at one time cover a narrow vocabulary window (W tiles are shared
//           through L2 by the token tiles) and each job keeps one candidate
//           list over its R tiles.  R = 1 is a plain vocabulary-strided walk.
//  RUNS     unit u owns token tile (u % m_tiles) over one contiguous
//           vocabulary range (range u / m_tiles of nr); the units owning one
//           range walk it in lockstep (W shared through L2) and each keeps
//           its candidate list across the whole range.
// The host picks the schedule with the fewest tiles on the busiest unit,
// charging short runs a little for their candidate-list restarts.
enum { SCHED_BLOCKS = 0, SCHED_RUNS = 1 };

struct Params {
  int M, V, d;
  int num_kc;        // K stages per tile = ceil(d / 64)
  int stages;        // shared-memory ring depth
  int a_box;         // A rows this CTA loads per stage (STREAM: M rounded up to 16)
  int a_stage_bytes;
  int b_rows;        // B rows this CTA loads per full tile (its half in a pair)
  int b_stage_bytes;
  int tmem_cols;
  // STREAM
  int units;         // 16-row vocabulary units
  // LARGE
  int m_tiles, v_tiles;  // token tiles of 128 rows (256 for pairs), vocabulary tiles of 256
  int sched;
  int nr;            // RUNS: vocabulary ranges per token tile
  int R;             // BLOCKS: vocabulary tiles per job
  int n_vblocks;     // BLOCKS: ceil(v_tiles / R)
  int b_widths[4];   // STREAM: the tile widths, one tensor map each
  int merge_halves;  // one run per unit: the two column halves merge in-kernel
  int store_only;    // plain GEMM: write z to z_dbg, no log-softmax / top-16
  int v_offset;      // added to every vocabulary index written to a record
  int w_prefetch;    // STREAM: K stages of W prefetched into L2 before the dependency wait
  int ksplit;        // plain GEMM, STREAM: CTAs per tile range, each over 1/ksplit of K
                     // (partial sums added into z_dbg, which the host zeroes first)
  int tail_units;    // STREAM: 16-row units of the narrow last tile of a long range (0: none)
  // outputs
  Partial* part;     // [M][P]
  int P;
  float* z_dbg;      // optional raw logits [M][V]
  int* status;
  unsigned long long timeout_ns;
};

// A record with the vocabulary indices shifted by `off` (a shard's first row).
__device__ __forceinline__ void store_record(Partial* dst, const TopState& st, int off) {
  int gi[KTOP];
#pragma unroll
  for (int k = 0; k < KTOP; ++k) gi[k] = st.i[k] == 0x7fffffff ? st.i[k] : st.i[k] + off;
  store_partial(dst, st.m, st.s, st.v, gi);
}

struct SmemLayout {
  uint32_t a, b, bars, misc, total;
};

// STREAM: how a CTA's range of n 16-row units is cut into tiles.  A range of
// at least tail + 16 units ends with a narrow tile of `tail` units, so that
// little epilogue work remains once the range's last weights have arrived;
// the rest is cut into the fewest tiles of at most 256 rows, all of (nearly)
// equal width (every tile costs a full K loop of MMAs whatever its width, so
// no tile is a sliver).  nt main tiles of wu units (the last may be
// narrower), then the tail.
struct StreamSplit {
  int nt, wu, tail;
};

__host__ __device__ inline StreamSplit stream_split(int n, int tail_units) {
  StreamSplit q;
  q.tail = (tail_units > 0 && n >= tail_units + TILE_N / 16) ? tail_units : 0;
  const int main_units = n - q.tail;
  q.nt = (main_units + TILE_N / 16 - 1) / (TILE_N / 16);
  q.wu = q.nt > 0 ? (main_units + q.nt - 1) / q.nt : 0;
  return q;
}

__host__ __device__ inline SmemLayout smem_layout(const Params& p) {
  SmemLayout s;
  s.a = 0;
  s.b = s.a + p.stages * p.a_stage_bytes;
  // an MMA reads a full 128-row span from its A stage: keep that span inside
  // the allocation (rows beyond the loaded box are never read back)
  uint32_t b_min = (p.stages - 1) * p.a_stage_bytes + MMA_A_SPAN;
  if (s.b < b_min) s.b = (b_min + 1023) & ~1023u;
  s.bars = s.b + p.stages * p.b_stage_bytes;
  s.misc = s.bars + (2 * p.stages + 6) * 8;
  s.total = s.misc + 16;
  return s;
}

// ------------------------------------------------------------ tile walks ---

template <bool PAIR>
__device__ __forceinline__ int unit_id() { return PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x); }
template <bool PAIR>
__device__ __forceinline__ int unit_count() { return PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x); }

struct Tile {
  int a_row;   // first token row of this CTA's A rows (and of its TMEM lanes)
  int b_row;   // first W row this CTA loads
  int n_cols;  // MMA N (vocabulary rows of the tile)
  int v0;      // vocabulary index of accumulator column 0
  int slot;    // partial-record slot of the tile's run
  bool first, last;
};

// The k-th tile of this CTA; false past the end.
template <int MODE, bool PAIR>
__device__ __forceinline__ bool get_tile(const Params& p, int k, uint32_t rank, Tile& t) {
  if (MODE == MODE_STREAM) {
    // The CTA's range of 16-row units, cut as stream_split says.
    const long long G = gridDim.x / p.ksplit, c = blockIdx.x % G;
    const int u0 = static_cast<int>((c * p.units) / G);
    const int u1 = static_cast<int>(((c + 1) * p.units) / G);
    const StreamSplit q = stream_split(u1 - u0, p.tail_units);
    const int main_end = u1 - q.tail;                    // first unit of the tail
    int t0, t1;
    if (k < q.nt) {
      t0 = u0 + k * q.wu;
      if (t0 >= main_end) return false;
      t1 = min(t0 + q.wu, main_end);
    } else if (k == q.nt && q.tail > 0) {
      t0 = main_end;
      t1 = u1;
    } else {
      return false;
    }
    t.a_row = 0;
    t.b_row = t0 * 16;
    t.n_cols = (t1 - t0) * 16;
    t.v0 = t0 * 16;
    t.slot = blockIdx.x;
    t.first = k == 0;
    t.last = t1 == u1;
    return true;
  }
  const int u = unit_id<PAIR>();
  int mt, vt;
  if (p.sched == SCHED_RUNS) {
    mt = u % p.m_tiles;
    const int r = u / p.m_tiles;
    const int lo = static_cast<int>(static_cast<long long>(r) * p.v_tiles / p.nr);
    const int hi = static_cast<int>(static_cast<long long>(r + 1) * p.v_tiles / p.nr);
    vt = lo + k;
    if (vt >= hi) return false;
    t.slot = r;
    t.first = k == 0;
    t.last = vt == hi - 1;
  } else {
    // k-th tile of this unit: job j = u + (k / R') * units ... walked job by
    // job; each job covers R tiles (the last vocabulary block may be shorter)
    const long long jobs = static_cast<long long>(p.m_tiles) * p.n_vblocks;
    long long job = u;
    int kk = k;
    for (;;) {
      if (job >= jobs) return false;
      const int vb = static_cast<int>(job / p.m_tiles);
      const int len = min(p.R, p.v_tiles - vb * p.R);
      if (kk < len) {
        mt = static_cast<int>(job - static_cast<long long>(vb) * p.m_tiles);
        vt = vb * p.R + kk;
        t.slot = vb;
        t.first = kk == 0;
        t.last = kk == len - 1;
        break;
      }
      kk -= len;
      job += unit_count<PAIR>();
    }
  }
  t.a_row = mt * (PAIR ? 2 * A_ROWS : A_ROWS) + static_cast<int>(rank) * A_ROWS;
  t.b_row = vt * TILE_N + static_cast<int>(rank) * p.b_rows;
  t.n_cols = TILE_N;
  t.v0 = vt * TILE_N;
  return true;
}

// ------------------------------------------------------------ epilogue -----

// Fold one 16-column chunk of a token row's logits (x[jj] is vocabulary index
// vbase + jj; the first nvalid are real) into the row's running
// (max, sum exp) and sorted top-16.  Called by a whole warp (one row per
// lane): candidates that can enter a lane's list are inserted by that lane,
// so the warp loops max over lanes of their count; an empty list (a run's
// first chunk) is filled by sorting the chunk.  Written for instruction-level
// parallelism: the max, the sum of exponentials and the candidate mask are
// trees over independent values, not chains through one accumulator, and a
// candidate's value is picked by a 4-level select tree.
__device__ __forceinline__ void fold_chunk(TopState& st, const float (&x)[16], int vbase, int nvalid) {
  float xv[16];
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) xv[jj] = jj < nvalid ? x[jj] : -INFINITY;
  float t8[8], t4[4];
#pragma unroll
  for (int q = 0; q < 8; ++q) t8[q] = fmaxf(xv[2 * q], xv[2 * q + 1]);
#pragma unroll
  for (int q = 0; q < 4; ++q) t4[q] = fmaxf(t8[2 * q], t8[2 * q + 1]);
  const float cmax = fmaxf(fmaxf(t4[0], t4[1]), fmaxf(t4[2], t4[3]));
  if (cmax > st.m) {
    st.s *= __expf(st.m - cmax);
    st.m = cmax;
  }
  float e[16];
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) e[jj] = __expf(xv[jj] - st.m);   // exp(-inf) = 0 for the padding
#pragma unroll
  for (int q = 0; q < 8; ++q) e[q] = e[2 * q] + e[2 * q + 1];
#pragma unroll
  for (int q = 0; q < 4; ++q) e[q] = e[2 * q] + e[2 * q + 1];
  st.s += (e[0] + e[1]) + (e[2] + e[3]);
  uint32_t pend = 0;
  if (nvalid == 16 && st.v[0] == -INFINITY) {
    st.assign_sorted16(x, vbase);
  } else {
    // a candidate must beat this list's 16th entry
    const float thr = st.v[KTOP - 1];
    uint32_t b4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      b4[q] = (xv[4 * q] > thr ? 1u : 0u) | (xv[4 * q + 1] > thr ? 2u : 0u) | (xv[4 * q + 2] > thr ? 4u : 0u) |
              (xv[4 * q + 3] > thr ? 8u : 0u);
    pend = (b4[0] | (b4[1] << 4)) | ((b4[2] << 8) | (b4[3] << 12));
  }
  while (__any_sync(0xffffffffu, pend != 0)) {
    if (pend) {
      const int jj = __ffs(pend) - 1;
      pend &= pend - 1;
      float s8[8], s4[4], s2[2];
#pragma unroll
      for (int q = 0; q < 8; ++q) s8[q] = (jj & 1) ? x[2 * q + 1] : x[2 * q];
#pragma unroll
      for (int q = 0; q < 4; ++q) s4[q] = (jj & 2) ? s8[2 * q + 1] : s8[2 * q];
#pragma unroll
      for (int q = 0; q < 2; ++q) s2[q] = (jj & 4) ? s4[2 * q + 1] : s4[2 * q];
      st.insert_scan((jj & 8) ? s2[1] : s2[0], vbase + jj);
    }
  }
}

// First K stage of this CTA's share of K (split only for the plain GEMM in
// STREAM mode: CTAs [ks*G, (ks+1)*G) take the ks-th of ksplit slices).
__device__ __forceinline__ int kc0_of(const Params& p) {
  const int ks = static_cast<int>(blockIdx.x / (gridDim.x / p.ksplit));
  return ks * p.num_kc / p.ksplit;
}

// ------------------------------------------------------------ kernel -------

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    lmhead_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_w2,
                  const __grid_constant__ CUtensorMap tm_w3, const Params p) {
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
  // pair: the other CTA hands its count of stage loads to the leader here
  const uint32_t handover_bar = bar0 + 8u * (2 * p.stages + 5);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  volatile int* peer_issued = reinterpret_cast<volatile int*>(smem + L.misc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  // a wait that gives up in one CTA of a pair stops the other one too
  const uint32_t peer_abort = PAIR ? mapa_shared(smem_addr(const_cast<int*>(abort_flag)), rank ^ 1u) : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PAIR ? 2 * EPI_THREADS : EPI_THREADS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(handover_bar, 1);
    *abort_flag = 0;
    *peer_issued = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if (MODE == MODE_STREAM) {
      prefetch_tmap(&tm_w1);
      prefetch_tmap(&tm_w2);
      prefetch_tmap(&tm_w3);
    }
  }
  if (warp == 1) {
    if (PAIR)
      tmem_alloc_pair(smem_addr(tmem_slot), p.tmem_cols);
    else
      tmem_alloc(smem_addr(tmem_slot), p.tmem_cols);
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (MODE == MODE_STREAM && warp == 0 && lane == 0) {
    // W is a weight the stream's previous kernels do not produce: start
    // pulling this CTA's first K stages of it into L2 while that kernel
    // finishes (an L2 prefetch fills no shared memory, so it cannot observe
    // anything stale).
    Tile t0;
    if (get_tile<MODE, PAIR>(p, 0, rank, t0)) {
      const CUtensorMap* mb = &tm_b;
      if (t0.n_cols == p.b_widths[1]) mb = &tm_w1;
      else if (t0.n_cols == p.b_widths[2]) mb = &tm_w2;
      else if (t0.n_cols == p.b_widths[3]) mb = &tm_w3;
      const int kc_end = min(kc0_of(p) + p.w_prefetch, p.num_kc);
      for (int kc = kc0_of(p); kc < kc_end; ++kc) tma_prefetch_l2_2d(mb, kc * BK, t0.b_row);
    }
  }
  // Set-up above overlaps the previous kernel; global memory (other than the
  // L2 prefetch of W) only from here.
  pdl_wait();
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  // this CTA's share of K (split only for the plain GEMM in STREAM mode)
  const int ks = MODE == MODE_STREAM ? static_cast<int>(blockIdx.x / (gridDim.x / p.ksplit)) : 0;
  const int kc0 = kc0_of(p);
  const int kc1 = (ks + 1) * p.num_kc / p.ksplit;

  int issued = 0;   // producer: stage loads issued, in ring order (load k went to stage k % stages)
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      const uint64_t pol_normal = l2_policy_evict_normal();
      // W is read once when streaming; shared by concurrent token tiles otherwise
      const uint64_t pol_w = MODE == MODE_STREAM ? pol_stream : pol_normal;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto load = [&](uint32_t dst, const CUtensorMap* m, uint32_t fb, int c0, int c1, uint64_t pol) {
        if (PAIR)
          tma_load_2d_pair(dst, m, mapa_shared(fb, 0), c0, c1, pol);
        else
          tma_load_2d_hint(dst, m, fb, c0, c1, pol);
      };
      Tile t;
      for (int k = 0; ok && get_tile<MODE, PAIR>(p, k, rank, t); ++k) {
        // bytes landing on the leader's barrier per stage (both CTAs of a pair)
        const int b_rows_here = MODE == MODE_STREAM ? t.n_cols : p.b_rows;
        const uint32_t tx = static_cast<uint32_t>((PAIR ? 2 : 1) * (p.a_box + b_rows_here) * BK * 2);
        for (int kc = kc0; kc < kc1; ++kc) {
          if (!mbar_wait(empty_bar(s), ph ^ 1u, deadline, abort_flag, p.status, peer_abort)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(s);
          if (leader) mbar_arrive_expect_tx(fb, tx);
          load(sbase + L.a + s * p.a_stage_bytes, &tm_a, fb, kc * BK, t.a_row, pol_keep);
          const uint32_t b_dst = sbase + L.b + s * p.b_stage_bytes;
          // one box per stage: the map whose box height is this tile's width
          // (STREAM tiles take one of at most four widths, known on the host)
          const CUtensorMap* mb = &tm_b;   // LARGE: the full tile; STREAM: width b_widths[0]
          if (MODE == MODE_STREAM) {
            if (b_rows_here == p.b_widths[1]) mb = &tm_w1;
            else if (b_rows_here == p.b_widths[2]) mb = &tm_w2;
            else if (b_rows_here == p.b_widths[3]) mb = &tm_w3;
          }
          load(b_dst, mb, fb, kc * BK, t.b_row, pol_w);
          ++issued;
          if (++s == p.stages) { s = 0; ph ^= 1u; }
        }
      }
      // pair: the other CTA hands the leader its count of loads (always: it
      // cannot know whether the leader will need it; see the drain below)
      if (PAIR && !leader) {
        st_shared_cluster_u32(mapa_shared(smem_addr(const_cast<int*>(peer_issued)), 0), static_cast<uint32_t>(issued));
        mbar_arrive_cluster(mapa_shared(handover_bar, 0));   // release: the count is visible first
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer ----
    if (lane == 0 && leader) {
      int s = 0;
      uint32_t ph = 0;
      int tb = 0;
      uint32_t tph = 0;
      bool ok = true;
      auto commit = [&](uint32_t bar) {
        if (PAIR)
          umma_commit_pair_multicast(bar, 0x3);
        else
          umma_commit(bar);
      };
      Tile t;
      for (int k = 0; ok && get_tile<MODE, PAIR>(p, k, rank, t); ++k) {
        const uint32_t idesc = umma_idesc_bf16_f32(PAIR ? 2 * A_ROWS : A_ROWS, t.n_cols);
        if (!mbar_wait(tempty_bar(tb), tph ^ 1u, deadline, abort_flag, p.status, peer_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * TILE_N);
        for (int kc = kc0; kc < kc1; ++kc) {
          if (!mbar_wait(full_bar(s), ph, deadline, abort_flag, p.status, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = umma_desc_sw128(sbase + L.a + s * p.a_stage_bytes);
          const uint64_t bdesc = umma_desc_sw128(sbase + L.b + s * p.b_stage_bytes);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // advance the start address by kk * 32 bytes (encoded >> 4)
            const uint32_t acc = ((kc - kc0) | kk) != 0 ? 1u : 0u;
            if (PAIR)
              umma_bf16_pair(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, idesc, acc);
            else
              umma_bf16(d_tmem, adesc + 2ull * kk, bdesc + 2ull * kk, idesc, acc);
          }
          commit(empty_bar(s));
          if (++s == p.stages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        commit(tfull_bar(tb));
        if (++tb == 2) { tb = 0; tph ^= 1u; }
      }
      // Every MMA this thread issued has completed before TMEM is released.
      if (PAIR)
        umma_commit_pair(drain_bar);
      else
        umma_commit(drain_bar);
      const uint64_t dl = globaltimer_ns() + 50000000ull;
      while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() < dl) {
      }
    }
  } else {
    // ------------------------------------------------------ epilogue ------
    const int ew = warp - 2;                  // 0..7
    const int quarter = warp & 3;             // TMEM lanes this warp may access
    const int half = ew >> 2;                 // which half of the tile's columns
    const int trow = quarter * 32 + lane;     // accumulator row held by this thread
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    TopState st;
    st.reset();
    int tb = 0;
    uint32_t tph = 0;
    int run_slot = -1;   // merge_halves: slot of the completed run
    int run_row = p.M;   // merge_halves: this thread's token row in that run
    Tile t;
    for (int k = 0; get_tile<MODE, PAIR>(p, k, rank, t); ++k) {
      int ok = 0;
      if (lane == 0) ok = mbar_wait(tfull_bar(tb), tph, deadline, abort_flag, p.status, peer_abort) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      if (t.first) st.reset();
      const int row = t.a_row + trow;
      const int nch = t.n_cols / 16;
      const int split = (nch + 1) >> 1;
      // the two warps of a lane quarter split the columns; warps whose 32 rows
      // are all past M only hand the buffer back
      const int ch_begin = half ? split : 0;
      const int ch_end = t.a_row + quarter * 32 >= p.M ? 0 : (half ? nch : split);
      const uint32_t taddr = tmem_base + static_cast<uint32_t>(tb * TILE_N) + lane_off;
      for (int ch = ch_begin; ch < ch_end; ++ch) {
        const int c0 = ch * 16;
        const int vbase = t.v0 + c0;
        if (vbase >= p.V) break;
        float x[16];
        tmem_ld16(taddr + c0, x);
        tmem_ld_wait();
        const int nvalid = min(16, p.V - vbase);
        if (p.store_only) {
          if (row < p.M && p.ksplit > 1) {
            float* zr = p.z_dbg + static_cast<size_t>(row) * p.V + vbase;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              if (jj < nvalid) atomicAdd(zr + jj, x[jj]);
          } else if (row < p.M) {
            float* zr = p.z_dbg + static_cast<size_t>(row) * p.V + vbase;
            if (nvalid == 16 && (p.V & 3) == 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<float4*>(zr)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj)
                if (jj < nvalid) zr[jj] = x[jj];
            }
          }
          continue;
        }
        fold_chunk(st, x, vbase, nvalid);
        if (p.z_dbg && row < p.M) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (jj < nvalid) p.z_dbg[static_cast<size_t>(row) * p.V + vbase + jj] = x[jj];
        }
      }
      // release the TMEM buffer to the MMA issuer (the leader's barrier)
      tc_fence_before();
      if (PAIR && !leader)
        mbar_arrive_cluster(mapa_shared(tempty_bar(tb), 0));
      else
        mbar_arrive(tempty_bar(tb));
      if (++tb == 2) { tb = 0; tph ^= 1u; }
      if (t.last && !p.store_only) {
        if (p.merge_halves) {
          run_slot = t.slot;
          run_row = row;
        } else if (row < p.M)
          store_record(p.part + static_cast<size_t>(row) * p.P + 2 * t.slot + half, st, p.v_offset);
      }
    }
    if (p.merge_halves && !p.store_only) {
      // One run per unit: its pipeline has drained, so the B stages hold the
      // exchange.  The half-1 warp of each lane quarter publishes its lists,
      // the half-0 warp folds them into its own and writes one record.
      float* xs = reinterpret_cast<float*>(smem + L.b) + trow * 36;
      if (half == 1) {
        xs[0] = st.m;
        xs[1] = st.s;
#pragma unroll
        for (int k = 0; k < KTOP; ++k) {
          xs[2 + k] = st.v[k];
          xs[18 + k] = __int_as_float(st.i[k]);
        }
      }
      named_barrier_sync(1 + quarter, 64);
      if (half == 0 && run_slot >= 0 && run_row < p.M) {
        float ov[KTOP];
        int oi[KTOP];
#pragma unroll
        for (int k = 0; k < KTOP; ++k) {
          ov[k] = xs[2 + k];
          oi[k] = __float_as_int(xs[18 + k]);
        }
        st.merge_lse(xs[0], xs[1]);
        st.merge_bitonic(ov, oi);
        store_record(p.part + static_cast<size_t>(run_row) * p.P + run_slot, st, p.v_offset);
      }
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (PAIR) cluster_sync_all();  // every role of both CTAs is done: abort flags and counts are final
  if (warp == 0 && lane == 0 && leader && *abort_flag != 0) {
    // Never leave with copies in flight: after giving up, the loads that
    // were issued but never consumed must be seen to land before the CTA
    // (and, in a pair, the other CTA) may exit.  Every load of a pair
    // completes on the leader's barriers, so the leader drains both CTAs'
    // loads.  Both CTAs fill the stages in the same order and one runs at
    // most a ring ahead of the other (a stage is refilled only after both
    // its loads were consumed), so the two counts say which stage loads
    // only one CTA issued: for a load only the leader issued, the other
    // CTA's bytes will never come and are counted as arrived (complete_tx);
    // for one only the other CTA issued, the leader's arrival is made with
    // that CTA's bytes alone (arrive.expect_tx).  The last phase of every
    // stage then completes exactly when its last copy has landed.
    const uint64_t dl = globaltimer_ns() + 50000000ull;
    int n_all = issued;
    if (PAIR && mbar_try_wait_acq_cluster(handover_bar, 0)) {   // arrived before the cluster barrier
      const int n_peer = *peer_issued;
      const uint32_t peer_tx = static_cast<uint32_t>((p.a_box + p.b_rows) * BK * 2);
      const int k_lo = min(issued, n_peer), k_hi = max(issued, n_peer);
      for (int k = k_lo; k < k_hi; ++k) {
        if (issued > n_peer)
          mbar_complete_tx(full_bar(k % p.stages), peer_tx);
        else
          mbar_arrive_expect_tx(full_bar(k % p.stages), peer_tx);
      }
      n_all = k_hi;
    }
    for (int q = 0; q < p.stages && q < n_all; ++q) {
      const int k_last = q + ((n_all - 1 - q) / p.stages) * p.stages;   // last load into stage q
      const uint32_t par = static_cast<uint32_t>(k_last / p.stages) & 1u;
      while (!mbar_try_wait(full_bar(q), par) && globaltimer_ns() < dl) {
      }
    }
  }
  if (PAIR) {
    __syncwarp();
    cluster_sync_all();  // the other CTA stays resident until the leader's drain is done
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else
      tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// Fold a warp's 32 lists (one per lane, plus each lane's (max, sum exp)) into
// one: afterwards lane r < 16 holds entry r of the merged list and every lane
// holds the merged (m, s).  Five butterfly levels; at each, a lane takes its
// xor-partner's sorted list, keeps the 16 best of the two (the elementwise
// better of a[k] and b[15-k], a bitonic sequence) and re-sorts them with four
// half-cleaner stages.
__device__ __forceinline__ void ce_desc(float& va, int& ia, float& vb, int& ib) {
  const bool sw = better(vb, ib, va, ia);
  const float tv = va;
  const int ti = ia;
  va = sw ? vb : va;
  ia = sw ? ib : ia;
  vb = sw ? tv : vb;
  ib = sw ? ti : ib;
}

__device__ __forceinline__ void warp_merge(TopState& st, float& out_v, int& out_i) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, st.m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, st.s, off);
    st.merge_lse(m2, s2);
    float pv[KTOP];
    int pi[KTOP];
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      pv[k] = __shfl_xor_sync(0xffffffffu, st.v[k], off);
      pi[k] = __shfl_xor_sync(0xffffffffu, st.i[k], off);
    }
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      const bool take = better(pv[KTOP - 1 - k], pi[KTOP - 1 - k], st.v[k], st.i[k]);
      st.v[k] = take ? pv[KTOP - 1 - k] : st.v[k];
      st.i[k] = take ? pi[KTOP - 1 - k] : st.i[k];
    }
#pragma unroll
    for (int j = KTOP / 2; j >= 1; j >>= 1) {
#pragma unroll
      for (int k = 0; k < KTOP; ++k)
        if ((k & j) == 0) ce_desc(st.v[k], st.i[k], st.v[k + j], st.i[k + j]);
    }
  }
  const int lane = threadIdx.x & 31;
  out_v = -INFINITY;
  out_i = 0x7fffffff;
#pragma unroll
  for (int r = 0; r < KTOP; ++r) {
    if (lane == r) {
      out_v = st.v[r];
      out_i = st.i[r];
    }
  }
}

// Fold a lane's share of a row's partial records (q = first, first+step, ...)
// into its list; records are loaded one ahead so loads overlap the work.
__device__ __forceinline__ void fold_records(TopState& st, const Partial* base, int first, int step, int P) {
  if (first >= P) return;
  PartialRegs cur, nxt;
  cur.load(base + first);
  if (first + step < P) nxt.load(base + first + step);
  // the first record is already a sorted list: it becomes the starting state
  st.m = cur.m();
  st.s = cur.s();
  cur.lists(st.v, st.i);
  cur = nxt;
  for (int q = first + step; q < P; q += step) {
    if (q + step < P) nxt.load(base + q + step);
    st.merge_lse(cur.m(), cur.s());
    float rv[KTOP];
    int ri[KTOP];
    cur.lists(rv, ri);
    st.insert_sorted(rv, ri);
    cur = nxt;
  }
}

// Threshold-and-rank merge: one CTA per row, no serial list merging.
// Every record is a sorted list, so any 16 entries of the row bound its 16th
// best value from below.  Pass 1 merges the records' (m, s) and takes as that
// bound tau the 16th largest of the records' leading entries (the first J of
// each record, J = ceil(16 / P), so that there are at least 16 of them),
// found by counting for each leading entry how many are at least as large;
// tau is raised to the largest 16th entry of any one record if that is
// higher.  Pass 2 gathers every entry >= tau (a prefix of each record) into
// shared memory -- typically a few more than 16.  Pass 3 gives each gathered
// entry its rank under the full order (value descending, index ascending)
// by counting the entries ahead of it; the entries ranked 0..15 are the
// row's top-16.  Ranks are distinct because a vocabulary index appears in
// exactly one record.  If ties overflow the shared buffers, the CTA falls
// back to folding the records list by list.
constexpr int MR_CAP = 1024;

template <int NT, bool MULTI>
__global__ void __launch_bounds__(NT) merge_kernel_rank(const Partial* __restrict__ part, int M, int Pr, int nrank,
                                                        float* __restrict__ topk_logp,
                                                        int32_t* __restrict__ topk_idx,
                                                        float* __restrict__ lse) {
  constexpr int NW = NT / 32;
  __shared__ float cv[MR_CAP];
  __shared__ int ci[MR_CAP];
  __shared__ float red_m[NW], red_s[NW], red_t[NW];
  __shared__ float fv[NW][KTOP];
  __shared__ int fi[NW][KTOP];
  __shared__ int count, nhead;
  __shared__ float sh_lse, sh_tau;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int row = blockIdx.x;
  // records [nrank][M][Pr]: record q of this row is rank q / Pr's record q % Pr
  const int P = MULTI ? Pr * nrank : Pr;
  const Partial* base = part + static_cast<size_t>(row) * Pr;
  auto rec = [&](int q) -> const Partial* {
    if (!MULTI) return base + q;
    const int rk = q / Pr;
    return part + (static_cast<size_t>(rk) * M + row) * Pr + (q - rk * Pr);
  };
  pdl_wait();
  pdl_trigger();
  if (tid == 0) {
    count = 0;
    nhead = 0;
  }
  __syncthreads();
  const int J = P >= KTOP ? 1 : (KTOP + P - 1) / P;  // leading entries per record

  // pass 1: (m, s) of the row, the largest 16th entry, the leading entries.
  // With at most one record per thread the whole record is loaded here and
  // kept in registers for pass 2 (one round trip to memory instead of two).
  const bool one_each = P <= NT;
  PartialRegs mine;
  if (one_each && tid < P) mine.load(rec(tid));
  TopState st;  // only m and s are used
  st.m = -INFINITY;
  st.s = 0.f;
  float tau16 = -INFINITY;
  for (int q = tid; q < P; q += NT) {
    float v[KTOP];
    int ixs[KTOP];
    if (one_each) {
      mine.lists(v, ixs);
      st.merge_lse(mine.m(), mine.s());
    } else {
      const float* r = reinterpret_cast<const float*>(rec(q));
      const float4 h = __ldg(reinterpret_cast<const float4*>(r));
      st.merge_lse(h.x, h.y);
#pragma unroll
      for (int k = 0; k < KTOP; ++k) v[k] = __ldg(r + 4 + k);
    }
    tau16 = fmaxf(tau16, v[KTOP - 1]);
    const int pos = atomicAdd(&nhead, J);
    for (int j = 0; j < J; ++j)
      if (pos + j < MR_CAP) cv[pos + j] = v[j < KTOP ? j : KTOP - 1];
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, st.m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, st.s, off);
    st.merge_lse(m2, s2);
    tau16 = fmaxf(tau16, __shfl_xor_sync(0xffffffffu, tau16, off));
  }
  if (lane == 0) {
    red_m[w] = st.m;
    red_s[w] = st.s;
  }
  __syncthreads();
  // the 16th largest leading entry: the largest h with #{h' >= h} >= 16
  const int nh = nhead < MR_CAP ? nhead : MR_CAP;
  float th = -INFINITY;
  for (int c = tid; c < nh; c += NT) {
    const float h = cv[c];
    int ge = 0;
    for (int j = 0; j < nh; ++j) ge += cv[j] >= h ? 1 : 0;
    if (ge >= KTOP) th = fmaxf(th, h);
  }
  th = fmaxf(th, tau16);
#pragma unroll
  for (int off = 16; off; off >>= 1) th = fmaxf(th, __shfl_xor_sync(0xffffffffu, th, off));
  if (lane == 0) red_t[w] = th;
  __syncthreads();
  if (tid == 0) {
    float t = red_t[0];
    for (int k = 1; k < NW; ++k) {
      st.merge_lse(red_m[k], red_s[k]);
      t = fmaxf(t, red_t[k]);
    }
    sh_lse = st.m + logf(st.s);
    sh_tau = t;
  }
  __syncthreads();  // also: every read of the leading entries is done
  const float tau = sh_tau;
  const float row_lse = sh_lse;

  // pass 2: gather the entries >= tau (a prefix of each record)
  for (int q = tid; q < P; q += NT) {
    float v[KTOP];
    int ix[KTOP];
    if (one_each) {
      mine.lists(v, ix);
    } else {
      PartialRegs rr;
      rr.load(rec(q));
      rr.lists(v, ix);
    }
    int c = 0;
#pragma unroll
    for (int k = 0; k < KTOP; ++k) c += (v[k] >= tau && ix[k] != 0x7fffffff) ? 1 : 0;
    if (c) {
      const int pos = atomicAdd(&count, c);
#pragma unroll
      for (int k = 0; k < KTOP; ++k) {
        if (k < c && pos + k < MR_CAP) {
          cv[pos + k] = v[k];
          ci[pos + k] = ix[k];
        }
      }
    }
  }
  __syncthreads();
  const int n = count;
  float* out_v = topk_logp + static_cast<size_t>(row) * KTOP;
  int32_t* out_i = topk_idx + static_cast<size_t>(row) * KTOP;
  if (n <= MR_CAP) {
    // pass 3: rank of each gathered entry
    for (int c = tid; c < n; c += NT) {
      const float v = cv[c];
      const int ix = ci[c];
      int rank = 0;
      for (int j = 0; j < n; ++j) rank += better(cv[j], ci[j], v, ix) ? 1 : 0;
      if (rank < KTOP) {
        out_v[rank] = v - row_lse;
        out_i[rank] = ix;
      }
    }
    if (tid >= n && tid < KTOP) {  // fewer than 16 entries in the whole row
      out_v[tid] = -INFINITY;
      out_i[tid] = 0x7fffffff;
    }
  } else {
    // ties overflowed a buffer: fold the records list by list
    TopState fs;
    fs.reset();
    if (MULTI) {
      for (int q = tid; q < P; q += NT) {
        PartialRegs r;
        r.load(rec(q));
        fs.merge_lse(r.m(), r.s());
        float rv[KTOP];
        int ri[KTOP];
        r.lists(rv, ri);
        fs.merge_bitonic(rv, ri);
      }
    } else {
      fold_records(fs, base, tid, NT, P);
    }
    float v;
    int ix;
    warp_merge(fs, v, ix);
    if (lane < KTOP) {
      fv[w][lane] = v;
      fi[w][lane] = ix;
    }
    __syncthreads();
    if (w == 0) {
      TopState fin;
      fin.reset();
      for (int c = lane; c < NW * KTOP; c += 32) fin.insert(fv[c / KTOP][c % KTOP], fi[c / KTOP][c % KTOP]);
      warp_merge(fin, v, ix);
      if (lane < KTOP) {
        out_v[lane] = v - row_lse;
        out_i[lane] = ix;
      }
    }
  }
  if (tid == 0 && lse != nullptr) lse[row] = row_lse;
}

// ------------------------------------------------------------ host side ----

static int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Budget of every mbarrier wait of one launch.  DFLASH_TIMEOUT_NS, read at
// every call (a positive count of nanoseconds; a process may change it
// between calls), takes precedence over DFLASH_TIMEOUT_MS, read once per
// process; without either the budget is 2 s.
static unsigned long long timeout_ns_from_env() {
  if (const char* e = std::getenv("DFLASH_TIMEOUT_NS")) {
    const long long ns = std::atoll(e);
    if (ns > 0) return static_cast<unsigned long long>(ns);
  }
  static unsigned long long v = [] {
    const char* e = std::getenv("DFLASH_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms <= 0) ms = 2000;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return v;
}

// Tuning knobs, read at every call (unset: the defaults below).
static int env_int(const char* name, int dflt, int lo, int hi) {
  const char* e = std::getenv(name);
  if (e == nullptr || e[0] == 0) return dflt;
  int v = std::atoi(e);
  return v < lo ? lo : (v > hi ? hi : v);
}

// Pairs (2-CTA MMA) are used unless DFLASH_PAIR=0 (read at every call).
static bool pair_allowed() {
  const char* e = std::getenv("DFLASH_PAIR");
  return !(e != nullptr && e[0] == '0');
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

template <int MODE, bool PAIR>
static cudaError_t set_smem_attr() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(lmhead_kernel<MODE, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_BUDGET + 2048);
  });
  return err;
}

// Clusters of two that can be resident at once (0 when pairs cannot run).
template <int MODE>
static int max_pair_clusters() {
  static std::once_flag once;
  static int n = 0;
  std::call_once(once, [] {
    if (set_smem_attr<MODE, true>() != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = SMEM_BUDGET + 1024;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, lmhead_kernel<MODE, true>, &cfg) == cudaSuccess) n = c;
    cudaGetLastError();
  });
  return n;
}

struct Plan {
  int mode;
  bool pair;
  int grid;
  Params p;
  size_t smem;
};

// Deepest ring of `per_stage` bytes that fits the shared-memory budget.
static int fit_stages(Params& p, int cap) {
  int best = 0;
  for (int s = 2; s <= cap; ++s) {
    p.stages = s;
    if (smem_layout(p).total + 1024 <= static_cast<uint32_t>(SMEM_BUDGET)) best = s;
  }
  p.stages = best;
  return best;
}

// Narrow last tile of every weight-streaming range: 4 units = 64 vocabulary
// rows, or DFLASH_STREAM_TAIL units (read at every call; 0 = no tail).
static int stream_tail_units() {
  const char* e = std::getenv("DFLASH_STREAM_TAIL");
  if (e == nullptr) return 4;
  const int v = std::atoi(e);
  return v < 0 ? 0 : (v > 8 ? 8 : v);
}

static bool make_plan(int M, int V, int d, int sms, Plan& pl, bool store_only = false) {
  if (M < 1 || V < 16 || d < 8 || d % 8 != 0 || sms < 1) return false;
  Params& p = pl.p;
  p = Params{};
  p.M = M;
  p.V = V;
  p.d = d;
  p.num_kc = (d + BK - 1) / BK;
  p.tmem_cols = 2 * TILE_N;
  p.ksplit = 1;
  if (M <= A_ROWS) {
    pl.mode = MODE_STREAM;
    pl.pair = false;
    p.a_box = (M + 15) & ~15;
    p.a_stage_bytes = p.a_box * BK * 2;
    p.b_rows = TILE_N;
    p.b_stage_bytes = p.b_rows * BK * 2;
    p.units = (V + 15) / 16;
    pl.grid = p.units < sms ? p.units : sms;
    p.merge_halves = 1;
    p.P = pl.grid;
    // the widths STREAM tiles can take (see get_tile and stream_split): per
    // range length u (ranges differ by at most one unit), the main width,
    // the last main tile's remainder and the tail; one tensor map per width,
    // at most four -- a tail that would make a fifth width is dropped
    p.tail_units = store_only ? 0 : stream_tail_units();
    const int u_lo = p.units / pl.grid;
    for (;;) {
      int nw = 0;
      bool fits = true;
      for (int j = 0; j < 4; ++j) p.b_widths[j] = -1;
      for (int u = u_lo; u <= u_lo + 1 && fits; ++u) {
        if (u < 1) continue;
        const StreamSplit q = stream_split(u, p.tail_units);
        const int ws[3] = {16 * q.wu, 16 * (u - q.tail - (q.nt - 1) * q.wu), 16 * q.tail};
        for (int w : ws) {
          if (w <= 0) continue;
          bool have = false;
          for (int j = 0; j < nw; ++j) have = have || p.b_widths[j] == w;
          if (!have) {
            if (nw == 4) {
              fits = false;
              break;
            }
            p.b_widths[nw++] = w;
          }
        }
      }
      if (fits) break;
      if (p.tail_units == 0) return false;
      p.tail_units = 0;
    }
    if (fit_stages(p, 12) < 2) return false;
  } else {
    pl.mode = MODE_LARGE;
    const int clusters = pair_allowed() ? max_pair_clusters<MODE_LARGE>() : 0;
    pl.pair = clusters >= 1;
    p.a_box = A_ROWS;
    p.a_stage_bytes = A_ROWS * BK * 2;
    p.b_rows = pl.pair ? TILE_N / 2 : TILE_N;
    p.b_stage_bytes = p.b_rows * BK * 2;
    const int m_rows = pl.pair ? 2 * A_ROWS : A_ROWS;
    p.m_tiles = (M + m_rows - 1) / m_rows;
    p.v_tiles = (V + TILE_N - 1) / TILE_N;
    const int units = pl.pair ? (clusters < sms / 2 ? clusters : sms / 2) : sms;
    // cost = tiles on the busiest unit, with each job restart charged as a
    // fraction of a tile (its candidate list starts empty)
    const double restart = 0.15;
    double best = 1e30;
    int used = 1;
    int nr = units / p.m_tiles;
    if (nr > p.v_tiles) nr = p.v_tiles;
    if (nr >= 1) {
      const long long t_run = (p.v_tiles + nr - 1) / nr;
      const double c = t_run * (1.0 + restart / t_run);
      if (c < best) {
        best = c;
        p.sched = SCHED_RUNS;
        p.nr = nr;
        used = nr * p.m_tiles;
        p.merge_halves = 1;
        p.P = nr;
      }
    }
    const int force_r = env_int("DFLASH_SCHED_R", 0, 0, 64);
    for (int R = 1; R <= 64; R *= 2) {
      if (force_r > 0 && R != force_r) continue;
      const int nvb = (p.v_tiles + R - 1) / R;
      const long long jobs = static_cast<long long>(p.m_tiles) * nvb;
      const int u = static_cast<int>(jobs < units ? jobs : units);
      const long long t_blk = ((jobs + u - 1) / u) * R;
      const double c = t_blk * (1.0 + restart / R);
      if (c < best || force_r > 0) {
        best = c;
        p.sched = SCHED_BLOCKS;
        p.R = R;
        p.n_vblocks = nvb;
        p.nr = 0;
        used = u;
        p.merge_halves = 0;
        p.P = 2 * nvb;
      }
    }
    pl.grid = pl.pair ? 2 * used : used;
    if (fit_stages(p, 8) < 2) return false;
  }
  pl.smem = smem_layout(p).total + 1024;
  return true;
}

static size_t part_bytes(const Plan& pl) {
  return static_cast<size_t>(pl.p.M) * pl.p.P * sizeof(Partial);
}

template <int MODE, bool PAIR>
static cudaError_t launch_main(const Plan& pl, const CUtensorMap& ta, const CUtensorMap* tb, cudaStream_t st) {
  const cudaError_t e = set_smem_attr<MODE, PAIR>();
  if (e != cudaSuccess) return e;
  return launch_kernel_cluster(lmhead_kernel<MODE, PAIR>, dim3(pl.grid), dim3(NUM_THREADS), pl.smem, st,
                               PAIR ? 2 : 1, ta, tb[0], tb[1], tb[2], tb[3], pl.p);
}

static cudaError_t launch_merge(const Partial* part, int M, int Pr, int nrank, float* topk_logp,
                                int32_t* topk_idx, float* lse, cudaStream_t st) {
  const bool wide = static_cast<long long>(Pr) * nrank > 128;
  if (nrank == 1)
    return wide ? launch_kernel(merge_kernel_rank<256, false>, dim3(M), dim3(256), 0, st, part, M, Pr, 1, topk_logp,
                                topk_idx, lse)
                : launch_kernel(merge_kernel_rank<128, false>, dim3(M), dim3(128), 0, st, part, M, Pr, 1, topk_logp,
                                topk_idx, lse);
  return wide ? launch_kernel(merge_kernel_rank<256, true>, dim3(M), dim3(256), 0, st, part, M, Pr, nrank, topk_logp,
                              topk_idx, lse)
              : launch_kernel(merge_kernel_rank<128, true>, dim3(M), dim3(128), 0, st, part, M, Pr, nrank, topk_logp,
                              topk_idx, lse);
}

// records_only: run the GEMM + epilogue kernel alone (the records stay in ws
// for a later merge, e.g. after gathering every shard's records); v_offset is
// added to the records' vocabulary indices.
static int launch(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, float* topk_logp,
                  int32_t* topk_idx, float* lse, float* z_dbg, void* ws, size_t ws_bytes, int* dev_status,
                  void* stream, bool store_only = false, bool records_only = false, int v_offset = 0) {
  if (!H || !W || (!ws && !store_only)) return DFLASH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(H) & 15) || (reinterpret_cast<uintptr_t>(W) & 15) ||
      (reinterpret_cast<uintptr_t>(ws) & 255) || (store_only && (reinterpret_cast<uintptr_t>(z_dbg) & 15)))
    return DFLASH_ERR_INVALID_ARG;
  Plan pl;
  if (!make_plan(M, V, d, num_sms_current(), pl, store_only)) return DFLASH_ERR_INVALID_ARG;
  if (!store_only && ws_bytes < part_bytes(pl)) return DFLASH_ERR_WORKSPACE;
  Params& p = pl.p;
  p.part = static_cast<Partial*>(ws);
  p.store_only = store_only ? 1 : 0;
  p.v_offset = v_offset;
  if (store_only && pl.mode == MODE_STREAM) {
    // few tile ranges and a long K: split K over otherwise idle SMs
    const int sms = num_sms_current();
    int ks = 1;
    if (pl.grid * 2 <= sms && p.num_kc >= 8) {
      ks = sms / pl.grid;
      if (ks > p.num_kc / 4) ks = p.num_kc / 4;
      if (ks > 16) ks = 16;
      if (ks < 1) ks = 1;
    }
    p.ksplit = ks;
    pl.grid *= ks;
  }
  p.z_dbg = z_dbg;
  p.status = dev_status;
  p.timeout_ns = timeout_ns_from_env();
  p.w_prefetch = env_int("DFLASH_W_PREFETCH", 8, 0, 64);

  // W maps: the full tile box, then (STREAM) one box per other tile width
  CUtensorMap ta, tb[4];
  bool ok = make_map(&ta, H, M, d, p.a_box) &&
            make_map(&tb[0], W, V, d, pl.mode == MODE_STREAM ? p.b_widths[0] : p.b_rows);
  for (int j = 1; j < 4; ++j) {
    if (pl.mode == MODE_STREAM && p.b_widths[j] > 0)
      ok = ok && make_map(&tb[j], W, V, d, p.b_widths[j]);
    else
      tb[j] = tb[0];
  }
  if (!ok) return DFLASH_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (p.ksplit > 1 && cudaMemsetAsync(z_dbg, 0, static_cast<size_t>(M) * V * sizeof(float), st) != cudaSuccess)
    return DFLASH_ERR_CUDA;
  if (pl.mode == MODE_STREAM)
    e = launch_main<MODE_STREAM, false>(pl, ta, tb, st);
  else
    e = pl.pair ? launch_main<MODE_LARGE, true>(pl, ta, tb, st) : launch_main<MODE_LARGE, false>(pl, ta, tb, st);
  if (e != cudaSuccess) return DFLASH_ERR_CUDA;
  if (z_dbg == nullptr && !store_only && !records_only) {
    if (launch_merge(p.part, M, p.P, 1, topk_logp, topk_idx, lse, st) != cudaSuccess) return DFLASH_ERR_CUDA;
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

extern "C" int dflash_gemm_bf16(const dflash_bf16* A, const dflash_bf16* B, float* C, int M, int N, int K,
                                void* stream) {
  if (!C || N < 16) return DFLASH_ERR_INVALID_ARG;
  return dflash::lm::launch(A, B, M, N, K, nullptr, nullptr, nullptr, C, nullptr, 0, nullptr, stream, true);
}

extern "C" int dflash_lmhead_topk_records(int M, int V, int d) {
  dflash::lm::Plan pl;
  if (!dflash::lm::make_plan(M, V, d, dflash::lm::num_sms_current(), pl)) return 0;
  return pl.p.P;
}

extern "C" int dflash_lmhead_topk_partial(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d,
                                          int v_offset, void* records, size_t records_bytes, int* dev_status,
                                          void* stream) {
  if (!records || v_offset < 0) return DFLASH_ERR_INVALID_ARG;
  return dflash::lm::launch(H, W, M, V, d, nullptr, nullptr, nullptr, nullptr, records, records_bytes, dev_status,
                            stream, false, true, v_offset);
}

extern "C" int dflash_lmhead_topk_merge(const void* records, int M, int P, int nrank, int K, float* topk_logp,
                                        int32_t* topk_idx, float* lse, void* stream) {
  if (!records || !topk_logp || !topk_idx || K != dflash::KTOP || M < 1 || P < 1 || nrank < 1)
    return DFLASH_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(records) & 15) return DFLASH_ERR_INVALID_ARG;
  const cudaError_t e = dflash::lm::launch_merge(static_cast<const dflash::Partial*>(records), M, P, nrank, topk_logp,
                                                 topk_idx, lse, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
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
// with cudaGetSymbolAddress once per device and CUDA context, with that device
// current, on the first call made in that context (again after a
// cudaDeviceReset, which gives the device a new context and the array a new
// address).  That first call should therefore happen before any stream
// capture begins.
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
static void* g_static_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current CUDA context (nullptr if it cannot be read).
static void* current_context() {
  static CtxGetCurrentFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(ptr);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_static_scratch on the current device.  It is looked
// up once per (device, context): a context created after cudaDeviceReset
// (or after the primary context was released) holds the array at a new
// address, so the cached one is refreshed whenever the current context is
// not the one it was read in.
static int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DFLASH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  void* ctx = current_context();
  if (g_static_ptr[dev] == nullptr || ctx == nullptr || ctx != g_static_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return DFLASH_ERR_CUDA;
    g_static_ptr[dev] = p;
    g_static_ctx[dev] = current_context();  // the lookup may have just made the primary context current
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
