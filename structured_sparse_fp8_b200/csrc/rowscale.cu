// rowscale.cu -- per-token activation scales and per-channel weight scales.
//
// The per-tensor rule (scale = amax / 448, 1 when amax = 0; code =
// E4M3(RN_fp32(x / scale))) applied to each row on its own: per token for X
// (the SlideSparse summary's fused quantiser scales each token), per output
// channel for W (the roadmap's finer-grained scales for outlier layers).
// Rows are independent, so one warp owns a row and no grid-wide reduction
// is needed: the warp reads the row once for its amax and again (from L1)
// to encode it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "quant_common.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kRowWarps = 8;   // rows per CTA
constexpr int kRowBatch = 4;   // 16-byte loads in flight per lane

// amax bits (largest |x| pattern, NaN/Inf sorting above every finite value)
// of a bf16 row of nvec 8-element vectors, reduced over the warp.
__device__ __forceinline__ uint32_t row_amax_bits(const uint4 *row, int nvec, int lane) {
  uint32_t m2 = 0;
  for (int v = lane; v < nvec; v += 32 * kRowBatch) {
    uint4 w[kRowBatch];
#pragma unroll
    for (int u = 0; u < kRowBatch; ++u)
      w[u] = v + 32 * u < nvec ? __ldg(row + v + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kRowBatch; ++u) m2 = __vmaxu2(m2, absmax8x2(w[u]));
  }
  return __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
}

__device__ __forceinline__ float scale_of_amax(uint32_t amax) {
  return amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
}

__device__ __forceinline__ uint32_t code_of(uint32_t h, float s) {
  return e4m3_code(__fdiv_rn(bf16_bits_to_float(h & 0xFFFFu), s));
}

__global__ void __launch_bounds__(32 * kRowWarps)
    pertoken_quantize_kernel(const uint16_t *__restrict__ x, int64_t rows, int64_t cols,
                             uint8_t *__restrict__ q, float *__restrict__ scales, int32_t *status) {
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int nvec = static_cast<int>(cols / 8);
  const uint4 *row = reinterpret_cast<const uint4 *>(x + r * cols);
  const uint32_t amax = row_amax_bits(row, nvec, lane);
  const float s = scale_of_amax(amax);
  if (lane == 0) {
    scales[r] = s;
    if (amax >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
  }
  uint2 *out = reinterpret_cast<uint2 *>(q + r * cols);
  for (int v = lane; v < nvec; v += 32) {
    const uint4 w = __ldg(row + v);
    const uint32_t h[4] = {w.x, w.y, w.z, w.w};
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      lo |= (code_of(h[i], s) | code_of(h[i] >> 16, s) << 8) << (16 * i);
      hi |= (code_of(h[2 + i], s) | code_of(h[2 + i] >> 16, s) << 8) << (16 * i);
    }
    out[v] = make_uint2(lo, hi);
  }
}

// 2:4 prune (the selection of the per-tensor weight path: the two largest
// |w| of each group of 4, ties to the lower index) with one scale per row.
__global__ void __launch_bounds__(32 * kRowWarps)
    perchannel_prune_kernel(const uint16_t *__restrict__ w, int N, int K, uint8_t *__restrict__ values,
                            uint8_t *__restrict__ meta, float *__restrict__ scales, int32_t *status) {
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (n >= N) return;
  const int nvec = K / 8;
  const uint4 *row = reinterpret_cast<const uint4 *>(w + n * K);
  const uint32_t amax = row_amax_bits(row, nvec, lane);
  const float s = scale_of_amax(amax);
  if (lane == 0) {
    scales[n] = s;
    if (amax >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
  }
  uint32_t *vout = reinterpret_cast<uint32_t *>(values + n * (K / 2));
  uint8_t *mout = meta + n * (K / 8);
  for (int v = lane; v < nvec; v += 32) {  // one vector = two groups
    const uint4 wv = __ldg(row + v);
    const uint32_t h[8] = {wv.x & 0xFFFFu, wv.x >> 16, wv.y & 0xFFFFu, wv.y >> 16,
                           wv.z & 0xFFFFu, wv.z >> 16, wv.w & 0xFFFFu, wv.w >> 16};
    uint32_t out = 0, mb = 0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const uint32_t a[4] = {h[4 * g] & 0x7FFFu, h[4 * g + 1] & 0x7FFFu, h[4 * g + 2] & 0x7FFFu,
                             h[4 * g + 3] & 0x7FFFu};
      const uint32_t keep = keep2of4(a);
      const int i0 = __ffs(keep) - 1, i1 = __ffs(keep & (keep - 1)) - 1;
      mb |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * g);
      out |= (code_of(h[4 * g + i0], s) | code_of(h[4 * g + i1], s) << 8) << (16 * g);
    }
    vout[v] = out;
    mout[v] = static_cast<uint8_t>(mb);
  }
}

}  // namespace

cudaError_t launch_quantize_pertoken(const void *x, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                                     int32_t *status, cudaStream_t st) {
  const int64_t grid = (rows + kRowWarps - 1) / kRowWarps;
  pertoken_quantize_kernel<<<static_cast<unsigned>(grid), 32 * kRowWarps, 0, st>>>(
      static_cast<const uint16_t *>(x), rows, cols, q, scales, status);
  return cudaGetLastError();
}

cudaError_t launch_prune24_perchannel(const void *w, int N, int K, uint8_t *values, uint8_t *meta,
                                      float *scales, int32_t *status, cudaStream_t st) {
  const int grid = (N + kRowWarps - 1) / kRowWarps;
  perchannel_prune_kernel<<<grid, 32 * kRowWarps, 0, st>>>(static_cast<const uint16_t *>(w), N, K, values,
                                                             meta, scales, status);
  return cudaGetLastError();
}

}  // namespace sp24
