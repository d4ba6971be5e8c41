// Two-tap block-local convolution, bf16 streaming.
//
// "DFlash 2: Keep Drafting Parallel", section "a lightweight local
// convolution" (formula Conv_k(x)_t = k_{t,0} x_t + k_{t,1} x_{t-1}) and
// Figure 4: each position mixes with its predecessor inside the block and the
// first position reads the last verified token's representation.
//
// One thread owns 8 channels (one 16-byte vector) of one block and walks the
// block's P positions, keeping x_{t-1} in registers, so every input byte is
// read once and every output byte written once.  Consecutive threads own
// consecutive 16-byte vectors of a row: coalesced 512-byte warp transactions.
// The product a1*x_{t-1} of two bf16 values is exact in fp32; fmaf adds
// a0*x_t with one rounding; the result is rounded to nearest-even bf16.
#include <cuda_bf16.h>

#include "common.cuh"

namespace dflash {
namespace conv {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(f[2 * k]));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(f[2 * k + 1]));
    w[k] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

constexpr int UNROLL = 4;

__global__ void __launch_bounds__(256) conv2tap_kernel(const uint4* __restrict__ x, const uint4* __restrict__ prev,
                                                       const uint4* __restrict__ a0, const uint4* __restrict__ a1,
                                                       uint4* __restrict__ y, int B, int P, int d8) {
  pdl_wait();
  pdl_trigger();
  const long long total = static_cast<long long>(B) * d8;
  for (long long id = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; id < total;
       id += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(id / d8);
    const int c = static_cast<int>(id - static_cast<long long>(b) * d8);
    float k0[8], k1[8], xp[8];
    unpack8(__ldg(a0 + c), k0);
    unpack8(__ldg(a1 + c), k1);
    if (prev != nullptr) {
      unpack8(__ldg(prev + static_cast<size_t>(b) * d8 + c), xp);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) xp[k] = 0.f;
    }
    const uint4* xb = x + static_cast<size_t>(b) * P * d8 + c;
    uint4* yb = y + static_cast<size_t>(b) * P * d8 + c;
    int t = 0;
    for (; t + UNROLL <= P; t += UNROLL) {
      uint4 in[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) in[u] = __ldcs(xb + static_cast<size_t>(t + u) * d8);
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        float xt[8], out[8];
        unpack8(in[u], xt);
#pragma unroll
        for (int k = 0; k < 8; ++k) out[k] = fmaf(k0[k], xt[k], k1[k] * xp[k]);
        __stcs(yb + static_cast<size_t>(t + u) * d8, pack8(out));
#pragma unroll
        for (int k = 0; k < 8; ++k) xp[k] = xt[k];
      }
    }
    for (; t < P; ++t) {
      float xt[8], out[8];
      unpack8(__ldcs(xb + static_cast<size_t>(t) * d8), xt);
#pragma unroll
      for (int k = 0; k < 8; ++k) out[k] = fmaf(k0[k], xt[k], k1[k] * xp[k]);
      __stcs(yb + static_cast<size_t>(t) * d8, pack8(out));
#pragma unroll
      for (int k = 0; k < 8; ++k) xp[k] = xt[k];
    }
  }
}

// Dynamic taps: tap j of channel c at (b, t) is a_j[c] + delta[(b*P+t), j*G + c/16]
// (corrections computed beforehand by the tensor-core GEMM).  A thread's 8
// channels lie in one 16-channel group.
__global__ void __launch_bounds__(256) conv2tap_dynamic_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ prev, const uint4* __restrict__ a0,
    const uint4* __restrict__ a1, const float* __restrict__ delta, uint4* __restrict__ y, int B, int P, int d8, int G) {
  pdl_wait();
  pdl_trigger();
  const long long total = static_cast<long long>(B) * d8;
  for (long long id = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; id < total;
       id += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(id / d8);
    const int c = static_cast<int>(id - static_cast<long long>(b) * d8);
    const int g = c >> 1;
    float k0[8], k1[8], xp[8];
    unpack8(__ldg(a0 + c), k0);
    unpack8(__ldg(a1 + c), k1);
    if (prev != nullptr) {
      unpack8(__ldg(prev + static_cast<size_t>(b) * d8 + c), xp);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) xp[k] = 0.f;
    }
    const uint4* xb = x + static_cast<size_t>(b) * P * d8 + c;
    uint4* yb = y + static_cast<size_t>(b) * P * d8 + c;
    const float* db = delta + static_cast<size_t>(b) * P * 2 * G + g;
    for (int t = 0; t < P; ++t) {
      float xt[8], out[8];
      unpack8(__ldcs(xb + static_cast<size_t>(t) * d8), xt);
      const float d0 = __ldg(db + static_cast<size_t>(t) * 2 * G);
      const float d1 = __ldg(db + static_cast<size_t>(t) * 2 * G + G);
#pragma unroll
      for (int k = 0; k < 8; ++k) out[k] = fmaf(k0[k] + d0, xt[k], (k1[k] + d1) * xp[k]);
      __stcs(yb + static_cast<size_t>(t) * d8, pack8(out));
#pragma unroll
      for (int k = 0; k < 8; ++k) xp[k] = xt[k];
    }
  }
}

}  // namespace conv
}  // namespace dflash

extern "C" int dflash_conv2tap(const dflash_bf16* x, const dflash_bf16* prev, const dflash_bf16* a0,
                               const dflash_bf16* a1, dflash_bf16* y, int B, int P, int d, void* stream) {
  if (!x || !a0 || !a1 || !y || B < 1 || P < 1 || d < 8 || d % 8 != 0) return DFLASH_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(a0) |
                        reinterpret_cast<uintptr_t>(a1) | reinterpret_cast<uintptr_t>(y) |
                        reinterpret_cast<uintptr_t>(prev);
  if (mis & 15) return DFLASH_ERR_INVALID_ARG;
  const int d8 = d / 8;
  const long long total = static_cast<long long>(B) * d8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  const cudaError_t e = dflash::launch_kernel(
      dflash::conv::conv2tap_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
      static_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(prev),
      reinterpret_cast<const uint4*>(a0), reinterpret_cast<const uint4*>(a1), reinterpret_cast<uint4*>(y), B, P, d8);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

extern "C" size_t dflash_conv2tap_dynamic_workspace(int B, int P, int d) {
  if (B < 1 || P < 1 || d < 128 || d % 16 != 0) return 0;
  return static_cast<size_t>(B) * P * 2 * (d / 16) * sizeof(float);
}

extern "C" int dflash_conv2tap_dynamic(const dflash_bf16* x, const dflash_bf16* prev, const dflash_bf16* a0,
                                       const dflash_bf16* a1, const dflash_bf16* wc, dflash_bf16* y, int B, int P,
                                       int d, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !a0 || !a1 || !wc || !y || !ws || B < 1 || P < 1 || d < 128 || d % 16 != 0)
    return DFLASH_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(a0) |
                        reinterpret_cast<uintptr_t>(a1) | reinterpret_cast<uintptr_t>(y) |
                        reinterpret_cast<uintptr_t>(prev) | reinterpret_cast<uintptr_t>(wc) |
                        reinterpret_cast<uintptr_t>(ws);
  if (mis & 15) return DFLASH_ERR_INVALID_ARG;
  if (ws_bytes < dflash_conv2tap_dynamic_workspace(B, P, d)) return DFLASH_ERR_WORKSPACE;
  const int G = d / 16;
  float* delta = static_cast<float*>(ws);
  // delta[(b*P+t), :] = x[b,t,:] . Wc^T  on the tensor-core GEMM path
  int rc = dflash_gemm_bf16(x, wc, delta, B * P, 2 * G, d, stream);
  if (rc != DFLASH_OK) return rc;
  const int d8 = d / 8;
  const long long total = static_cast<long long>(B) * d8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (total + 255) / 256;
  if (blocks > static_cast<long long>(sms) * 8) blocks = static_cast<long long>(sms) * 8;
  const cudaError_t e = dflash::launch_kernel(
      dflash::conv::conv2tap_dynamic_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
      static_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(prev),
      reinterpret_cast<const uint4*>(a0), reinterpret_cast<const uint4*>(a1), static_cast<const float*>(delta),
      reinterpret_cast<uint4*>(y), B, P, d8, G);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
