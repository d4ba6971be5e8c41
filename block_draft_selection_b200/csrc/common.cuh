// Shared device helpers for the sm_100a kernels: status words, bounded
// mbarrier waits, TMA tile loads, tcgen05 (TMEM / UMMA) wrappers.
//
// Every wait here is bounded by a deadline on %globaltimer.  A wait that runs
// out records DFLASH_ERR_TIMEOUT in the caller's status word and returns
// false; the calling role then drains what it has in flight and leaves, so
// no kernel in this library can spin forever.
#pragma once

#include <cstdint>
#include <cstdlib>
#include <utility>

#include <cuda_runtime.h>

#include "../../include/dflash.h"

#ifndef __CUDACC_RTC__
#include <cuda.h>
#endif

namespace dflash {

// ---------------------------------------------------------------- status ---

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------- programmatic dependent launch --
// Every kernel of the library waits for its stream predecessor before it
// touches global memory (a no-op when launched without the PDL attribute) and
// lets its own dependents begin launching once it no longer needs to be
// ahead of them.  Launch latency of the next kernel then overlaps this one.

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// On unless DFLASH_PDL=0 (read at every launch, so a caller can capture one
// graph with and another without programmatic launch).
inline bool pdl_enabled() {
  const char* e = std::getenv("DFLASH_PDL");
  return !(e != nullptr && e[0] == '0');
}

// Launch with programmatic stream serialisation (and an optional cluster
// size) through cudaLaunchKernelEx.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Same, launched as clusters of `cluster_x` consecutive CTAs along x (no
// cluster attribute when cluster_x == 1).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                         cudaStream_t st, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- mbarrier --

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with acquire at cluster scope: what another CTA of the cluster
// wrote before its release-arrive on this barrier is visible afterwards.
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Store a 32-bit value into another CTA's shared memory (a shared::cluster
// address from mapa).
__device__ __forceinline__ void st_shared_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Wait for the phase with the given parity to complete, at most until
// `deadline` (globaltimer ns) or until *abort becomes nonzero.  Returns false
// (and records a timeout) when it gives up.  A nonzero `peer_abort` (the
// shared::cluster address of the other CTA's abort flag in a pair) is set
// too, so both CTAs of a pair stop together.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t deadline,
                                          volatile int* abort, int* status, uint32_t peer_abort = 0) {
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++spins & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() > deadline) {
        set_status(status, DFLASH_ERR_TIMEOUT);
        *abort = 1;
        if (peer_abort != 0) st_shared_cluster_u32(peer_abort, 1u);
        return false;
      }
    }
  }
  return true;
}

// Count `bytes` as arrived on the barrier's current phase without a copy
// (the transaction count drops as if they had landed).
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- TMA -------

// 2-D tiled bulk tensor load global -> shared, completion counted in bytes on
// `bar`.  c0 is the innermost (contiguous) coordinate in elements, c1 the row.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// Same, with an L2 eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Bring a 2-D tile of a tensor into L2 only (no shared memory, no barrier).
// Safe to issue before the stream predecessor has finished: L2 is the point
// of coherence, so a later write by that predecessor updates the line.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05 ---

// Shared-memory matrix descriptor for a K-major bf16 operand laid out by a
// 128-byte-swizzled TMA load: rows of 128 bytes (64 bf16), 8-row swizzle
// atoms of 1024 bytes stacked along M/N.  Fields (tcgen05 matrix descriptor):
// [0,14) start address >> 4; [16,30) leading byte offset >> 4 (unused for
// swizzled K-major, set to 1); [32,46) stride byte offset >> 4 (1024 B between
// 8-row atoms); [46,48) descriptor version = 1; [49,52) base offset = 0
// (atoms are 1024-byte aligned); [61,64) swizzle mode 2 = 128-byte.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor for tcgen05.mma kind::f16 with bf16 A and B, fp32
// accumulate, both operands K-major, dense: [4,6) D format (1 = f32);
// [7,10) A format (1 = bf16); [10,13) B format (1 = bf16); bits 15/16 = 0
// (K-major); [17,23) N >> 3; [24,29) M >> 4.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread
// has completed (and its shared-memory operands may be overwritten).
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM allocation: executed by one full warp.  Writes the base address to
// *dst_smem.  ncols is a power of two in [32, 512].
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp receives
// TMEM lane (lane base + t), columns [col, col+16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ int elect_lane0() { return (threadIdx.x & 31) == 0; }

// ------------------------------------------------- 2-CTA (cta_group::2) ----
// A cluster of two CTAs shares one tcgen05.mma of M = 256: each CTA stages
// half of A (128 rows) and half of B (N/2 rows) in its own shared memory at
// the same offsets; the leader (rank 0) issues the MMA and each CTA's TMEM
// receives its 128 rows of D.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier of another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA load into this CTA's shared memory whose byte count completes on the
// leader's barrier (`bar_cluster` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at this offset in every CTA of `cta_mask` when
// the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair_multicast(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ------------------------------------------------------ top-16 in registers --

constexpr int KTOP = 16;

// (value desc, index asc) strict order.
__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// Running candidate list kept sorted in registers, plus an online
// log-sum-exp state (m = running max, s = sum of exp(z - m)).
struct TopState {
  float v[KTOP];
  int i[KTOP];
  float m;
  float s;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      v[k] = -INFINITY;
      i[k] = 0x7fffffff;
    }
    m = -INFINITY;
    s = 0.f;
  }

  // Insert (x, ix) if it beats the current 16th entry under the full order.
  // The list is sorted, so the entries that stay ahead of x form a prefix;
  // every slot's new content depends only on two compares of the old list,
  // so the 16 slots update in parallel (no serial bubble chain).
  __device__ __forceinline__ void insert(float x, int ix) {
    if (!better(x, ix, v[KTOP - 1], i[KTOP - 1])) return;
    bool ahead[KTOP];
#pragma unroll
    for (int k = 0; k < KTOP; ++k) ahead[k] = better(v[k], i[k], x, ix);
    float nv[KTOP];
    int ni[KTOP];
    nv[0] = ahead[0] ? v[0] : x;
    ni[0] = ahead[0] ? i[0] : ix;
#pragma unroll
    for (int k = 1; k < KTOP; ++k) {
      nv[k] = ahead[k] ? v[k] : (ahead[k - 1] ? x : v[k - 1]);
      ni[k] = ahead[k] ? i[k] : (ahead[k - 1] ? ix : i[k - 1]);
    }
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      v[k] = nv[k];
      i[k] = ni[k];
    }
  }

  // Insert for a scan that visits indices in increasing order: any entry
  // already in the list has a smaller index than `ix`, so an equal value stays
  // ahead and every order test is a single value compare.
  __device__ __forceinline__ void insert_scan(float x, int ix) {
    if (!(x > v[KTOP - 1])) return;
    bool ahead[KTOP];
#pragma unroll
    for (int k = 0; k < KTOP; ++k) ahead[k] = v[k] >= x;
    float nv[KTOP];
    int ni[KTOP];
    nv[0] = ahead[0] ? v[0] : x;
    ni[0] = ahead[0] ? i[0] : ix;
#pragma unroll
    for (int k = 1; k < KTOP; ++k) {
      nv[k] = ahead[k] ? v[k] : (ahead[k - 1] ? x : v[k - 1]);
      ni[k] = ahead[k] ? i[k] : (ahead[k - 1] ? ix : i[k - 1]);
    }
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      v[k] = nv[k];
      i[k] = ni[k];
    }
  }

  // Keep the 16 best of this list and another sorted list.  The elementwise
  // better of v[k] and o[15-k] holds exactly those 16 as a bitonic sequence
  // (one list descending against the other ascending); four half-cleaner
  // stages sort it.  48 compare-exchanges with static indices, no serial
  // insertion chain.
  __device__ __forceinline__ void merge_bitonic(const float (&ov)[KTOP], const int (&oi)[KTOP]) {
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      const bool take = better(ov[KTOP - 1 - k], oi[KTOP - 1 - k], v[k], i[k]);
      v[k] = take ? ov[KTOP - 1 - k] : v[k];
      i[k] = take ? oi[KTOP - 1 - k] : i[k];
    }
#pragma unroll
    for (int j = KTOP / 2; j >= 1; j >>= 1) {
#pragma unroll
      for (int k = 0; k < KTOP; ++k)
        if ((k & j) == 0) cex(k, k + j, true);
    }
  }

  // Make the list the 16 values x[jj] (indices base + jj), sorted by a
  // bitonic sorting network: the fast way to fill an empty list.
  __device__ __forceinline__ void assign_sorted16(const float (&x)[KTOP], int base) {
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      v[k] = x[k];
      i[k] = base + k;
    }
#pragma unroll
    for (int size = 2; size <= KTOP; size <<= 1) {
#pragma unroll
      for (int stride = size / 2; stride > 0; stride >>= 1) {
#pragma unroll
        for (int k = 0; k < KTOP; ++k) {
          const int partner = k ^ stride;
          if (partner > k) cex(k, partner, (k & size) == 0);
        }
      }
    }
  }

  // Compare-exchange entries a < b: desc puts the better one at a.
  __device__ __forceinline__ void cex(int a, int b, bool desc) {
    const bool sw = desc ? better(v[b], i[b], v[a], i[a]) : better(v[a], i[a], v[b], i[b]);
    const float tv = v[a];
    const int ti = i[a];
    v[a] = sw ? v[b] : v[a];
    i[a] = sw ? i[b] : i[a];
    v[b] = sw ? tv : v[b];
    i[b] = sw ? ti : i[b];
  }

  // Insert the entries of another sorted list while they beat the 16th entry.
  __device__ __forceinline__ void insert_sorted(const float (&ov)[KTOP], const int (&oi)[KTOP]) {
#pragma unroll
    for (int k = 0; k < KTOP; ++k) {
      if (!better(ov[k], oi[k], v[KTOP - 1], i[KTOP - 1])) break;
      insert(ov[k], oi[k]);
    }
  }

  // Fold another (m, s) pair into this one.
  __device__ __forceinline__ void merge_lse(float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
      m = m2;
      s = s2;
      return;
    }
    const float mn = fmaxf(m, m2);
    s = s * __expf(m - mn) + s2 * __expf(m2 - mn);
    m = mn;
  }

  // Remove the head (entry 0), shifting the list up; the tail becomes empty.
  __device__ __forceinline__ void pop_head() {
#pragma unroll
    for (int k = 0; k < KTOP - 1; ++k) {
      v[k] = v[k + 1];
      i[k] = i[k + 1];
    }
    v[KTOP - 1] = -INFINITY;
    i[KTOP - 1] = 0x7fffffff;
  }
};

// Partial record written per (row, slot) by the LM-head kernel and read by
// the merge kernel: running max, sum of exp(z - max), 16 candidates.
struct __align__(16) Partial {
  float m;
  float s;
  float pad[2];
  float v[KTOP];
  int i[KTOP];
};
static_assert(sizeof(Partial) == 144, "partial record layout");

// Store a list as one partial record with 16-byte stores.
__device__ __forceinline__ void store_partial(Partial* rec, float m, float s, const float (&v)[KTOP],
                                              const int (&i)[KTOP]) {
  float4* d = reinterpret_cast<float4*>(rec);
  d[0] = make_float4(m, s, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 4; ++q) d[1 + q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[5 + q] = make_float4(__int_as_float(i[4 * q]), __int_as_float(i[4 * q + 1]), __int_as_float(i[4 * q + 2]),
                           __int_as_float(i[4 * q + 3]));
}

// Load a partial record with 16-byte read-only loads.
struct PartialRegs {
  float4 q[9];
  __device__ __forceinline__ void load(const Partial* rec) {
    const float4* s = reinterpret_cast<const float4*>(rec);
#pragma unroll
    for (int k = 0; k < 9; ++k) q[k] = __ldg(s + k);
  }
  __device__ __forceinline__ float m() const { return q[0].x; }
  __device__ __forceinline__ float s() const { return q[0].y; }
  __device__ __forceinline__ void lists(float (&v)[KTOP], int (&i)[KTOP]) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[4 * k] = q[1 + k].x;
      v[4 * k + 1] = q[1 + k].y;
      v[4 * k + 2] = q[1 + k].z;
      v[4 * k + 3] = q[1 + k].w;
      i[4 * k] = __float_as_int(q[5 + k].x);
      i[4 * k + 1] = __float_as_int(q[5 + k].y);
      i[4 * k + 2] = __float_as_int(q[5 + k].z);
      i[4 * k + 3] = __float_as_int(q[5 + k].w);
    }
  }
};

}  // namespace dflash
