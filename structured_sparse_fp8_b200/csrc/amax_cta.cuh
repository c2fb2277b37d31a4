// amax_cta.cuh -- shared pieces of the two-launch quantisers (slide.cu,
// int8.cu): the first launch, the bf16 amax of a tensor reduced in each CTA
// and then by one atomic per CTA into a workspace word that starts at zero,
// and the departure count that ends the second launch.  Internal
// linkage: every source that includes it gets its own kernel.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "quant_common.cuh"

namespace sp24 {
namespace {

constexpr int kAmaxThreads = 512;
constexpr int kAmaxBatch = 4;  // 16-byte loads in flight per thread

// ws[0] <- max(ws[0], amax bits of x); x has nvec 8-element vectors.
__global__ void __launch_bounds__(kAmaxThreads)
    bf16_amax_kernel(const uint4 *__restrict__ x, int64_t nvec, uint32_t *ws) {
  __shared__ uint32_t s_red[kAmaxThreads / 32];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kAmaxThreads;
  uint32_t m2 = 0;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * kAmaxThreads + threadIdx.x; v < nvec;
       v += stride * kAmaxBatch) {
    uint4 w[kAmaxBatch];
#pragma unroll
    for (int u = 0; u < kAmaxBatch; ++u)
      w[u] = v + stride * u < nvec ? __ldg(x + v + stride * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kAmaxBatch; ++u) m2 = __vmaxu2(m2, absmax8x2(w[u]));
  }
  const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    const uint32_t r = __reduce_max_sync(0xFFFFFFFFu, threadIdx.x < kAmaxThreads / 32 ? s_red[threadIdx.x] : 0u);
    if (threadIdx.x == 0) atomicMax(&ws[0], r);
  }
}

// Grid for nvec vectors: enough CTAs for kAmaxBatch vectors per thread, at
// most `cap`.
inline unsigned bf16_amax_grid(int64_t nvec, int64_t cap) {
  const int64_t per = static_cast<int64_t>(kAmaxThreads) * kAmaxBatch;
  int64_t g = (nvec + per - 1) / per;
  if (g > cap) g = cap;
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

// End of the second launch: the last CTA to leave returns the two workspace
// words (ws[0] amax, ws[1] departures) to zero for the next call.
__device__ __forceinline__ void workspace_depart(uint32_t *ws) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&ws[1], 1u) == gridDim.x - 1) {
      ws[0] = 0u;
      ws[1] = 0u;
    }
  }
}

inline cudaError_t launch_bf16_amax(const void *x, int64_t nvec, uint32_t *ws, int64_t cap, cudaStream_t st) {
  bf16_amax_kernel<<<bf16_amax_grid(nvec, cap), kAmaxThreads, 0, st>>>(static_cast<const uint4 *>(x), nvec, ws);
  return cudaGetLastError();
}

}  // namespace
}  // namespace sp24
