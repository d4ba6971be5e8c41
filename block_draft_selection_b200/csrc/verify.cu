// Greedy verification: one warp per block.
//
// "DFlash 2: Keep Drafting Parallel", Table 1 caption: the accepted length
// includes the verifier's next token.  Lane i compares draft[b,i] with the
// target's argmax token at position i; the first differing lane (ballot +
// find-first-set) is n, accept_len = n + 1 and next_token = target[b, n]
// (n = L when all L positions match: the target's bonus token).
#include "common.cuh"

namespace dflash {
namespace ver {

constexpr int WARPS = 8;

__global__ void __launch_bounds__(32 * WARPS) verify_kernel(const int32_t* __restrict__ draft,
                                                             const int32_t* __restrict__ target, int B, int L,
                                                             int32_t* __restrict__ accept_len,
                                                             int32_t* __restrict__ next_token) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const bool differs = lane < L && draft[static_cast<size_t>(b) * L + lane] !=
                                       target[static_cast<size_t>(b) * (L + 1) + lane];
  const unsigned mask = __ballot_sync(0xffffffffu, differs);
  const int n = mask ? __ffs(mask) - 1 : L;
  if (lane == 0) {
    accept_len[b] = n + 1;
    next_token[b] = target[static_cast<size_t>(b) * (L + 1) + n];
  }
}

}  // namespace ver
}  // namespace dflash

extern "C" int dflash_verify(const int32_t* draft, const int32_t* target, int B, int L, int32_t* accept_len,
                             int32_t* next_token, void* stream) {
  using namespace dflash::ver;
  if (!draft || !target || !accept_len || !next_token || B < 1 || L < 1 || L > 32) return DFLASH_ERR_INVALID_ARG;
  const cudaError_t e = dflash::launch_kernel(verify_kernel, dim3((B + WARPS - 1) / WARPS), dim3(32 * WARPS), 0,
                                              static_cast<cudaStream_t>(stream), draft, target, B, L, accept_len,
                                              next_token);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
