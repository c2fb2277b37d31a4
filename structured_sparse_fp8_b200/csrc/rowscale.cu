// rowscale.cu -- per-token activation scales and per-channel weight scales.
//
// The per-tensor rule (scale = amax / 448, 1 when amax = 0; code =
// E4M3(RN_fp32(x / scale))) applied to each row on its own: per token for X
// (the SlideSparse summary's fused quantiser scales each token), per output
// channel for W (the roadmap's finer-grained scales for outlier layers).
// Rows are independent, so no grid-wide reduction is needed: one warp owns
// a row (many rows), or a whole CTA does (few or long rows, so that the grid
// still fills the SMs); it reads the row once for its amax and again (from
// L1) to encode it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "quant_common.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kRowWarps = 8;   // rows per CTA
constexpr int kRowBatch = 4;   // 16-byte loads in flight per lane

// A row is worked on by T threads (a warp, or the whole CTA); thread i of
// the group handles vectors i, i + T, ...
template <bool BLOCK>
struct RowGroup {
  static constexpr int kT = BLOCK ? 32 * kRowWarps : 32;
  int i;  // index in the group
  __device__ __forceinline__ RowGroup() : i(BLOCK ? static_cast<int>(threadIdx.x) : static_cast<int>(threadIdx.x & 31)) {}
  // largest of v over the group (unsigned)
  __device__ __forceinline__ uint32_t max_all(uint32_t v, uint32_t *s_red) const {
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    if constexpr (BLOCK) {
      if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
      __syncthreads();
      v = s_red[0];
#pragma unroll
      for (int w = 1; w < kRowWarps; ++w) v = max(v, s_red[w]);
    }
    return v;
  }
};

// amax bits (largest |x| pattern, NaN/Inf sorting above every finite value)
// of a bf16 row of nvec 8-element vectors, reduced over the group.
template <bool BLOCK>
__device__ __forceinline__ uint32_t row_amax_bits(const uint4 *row, int nvec, const RowGroup<BLOCK> &g,
                                                  uint32_t *s_red) {
  constexpr int T = RowGroup<BLOCK>::kT;
  uint32_t m2 = 0;
  for (int v = g.i; v < nvec; v += T * kRowBatch) {
    uint4 w[kRowBatch];
#pragma unroll
    for (int u = 0; u < kRowBatch; ++u)
      w[u] = v + T * u < nvec ? __ldg(row + v + T * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kRowBatch; ++u) m2 = __vmaxu2(m2, absmax8x2(w[u]));
  }
  return g.max_all(max(m2 & 0xFFFFu, m2 >> 16), s_red);
}

__device__ __forceinline__ float scale_of_amax(uint32_t amax) {
  return amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
}

__device__ __forceinline__ uint32_t code_of(uint32_t h, float s) {
  return e4m3_code(__fdiv_rn(bf16_bits_to_float(h & 0xFFFFu), s));
}

template <bool BLOCK>
__global__ void __launch_bounds__(32 * kRowWarps)
    pertoken_quantize_kernel(const uint16_t *__restrict__ x, int64_t rows, int64_t cols,
                             uint8_t *__restrict__ q, float *__restrict__ scales, int32_t *status) {
  __shared__ uint32_t s_red[kRowWarps];
  const RowGroup<BLOCK> grp;
  const int64_t r = BLOCK ? static_cast<int64_t>(blockIdx.x)
                          : static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int nvec = static_cast<int>(cols / 8);
  const uint4 *row = reinterpret_cast<const uint4 *>(x + r * cols);
  const uint32_t amax = row_amax_bits(row, nvec, grp, s_red);
  const float s = scale_of_amax(amax);
  if (grp.i == 0) {
    scales[r] = s;
    if (amax >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
  }
  uint2 *out = reinterpret_cast<uint2 *>(q + r * cols);
  for (int v = grp.i; v < nvec; v += RowGroup<BLOCK>::kT) {
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
template <bool BLOCK>
__global__ void __launch_bounds__(32 * kRowWarps)
    perchannel_prune_kernel(const uint16_t *__restrict__ w, int N, int K, uint8_t *__restrict__ values,
                            uint8_t *__restrict__ meta, float *__restrict__ scales, int32_t *status) {
  __shared__ uint32_t s_red[kRowWarps];
  const RowGroup<BLOCK> grp;
  const int64_t n = BLOCK ? static_cast<int64_t>(blockIdx.x)
                          : static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (n >= N) return;
  const int nvec = K / 8;
  const uint4 *row = reinterpret_cast<const uint4 *>(w + n * K);
  const uint32_t amax = row_amax_bits(row, nvec, grp, s_red);
  const float s = scale_of_amax(amax);
  if (grp.i == 0) {
    scales[n] = s;
    if (amax >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
  }
  uint32_t *vout = reinterpret_cast<uint32_t *>(values + n * (K / 2));
  uint8_t *mout = meta + n * (K / 8);
  for (int v = grp.i; v < nvec; v += RowGroup<BLOCK>::kT) {  // one vector = two groups
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

// A CTA per row when a warp per row would leave the SMs short of warps
// (fewer rows than ~16 warps per SM) or give each lane a long serial walk
// (more than 32 vectors of 8 per lane).
static bool block_per_row(int64_t rows, int64_t cols) {
  return rows < 16 * 148 || cols / 8 > 32 * 32;
}

cudaError_t launch_quantize_pertoken(const void *x, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                                     int32_t *status, cudaStream_t st) {
  const uint16_t *xx = static_cast<const uint16_t *>(x);
  if (block_per_row(rows, cols)) {
    pertoken_quantize_kernel<true><<<static_cast<unsigned>(rows), 32 * kRowWarps, 0, st>>>(xx, rows, cols, q,
                                                                                          scales, status);
  } else {
    const int64_t grid = (rows + kRowWarps - 1) / kRowWarps;
    pertoken_quantize_kernel<false><<<static_cast<unsigned>(grid), 32 * kRowWarps, 0, st>>>(xx, rows, cols, q,
                                                                                           scales, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_prune24_perchannel(const void *w, int N, int K, uint8_t *values, uint8_t *meta,
                                      float *scales, int32_t *status, cudaStream_t st) {
  const uint16_t *ww = static_cast<const uint16_t *>(w);
  if (block_per_row(N, K)) {
    perchannel_prune_kernel<true><<<N, 32 * kRowWarps, 0, st>>>(ww, N, K, values, meta, scales, status);
  } else {
    const int grid = (N + kRowWarps - 1) / kRowWarps;
    perchannel_prune_kernel<false><<<grid, 32 * kRowWarps, 0, st>>>(ww, N, K, values, meta, scales, status);
  }
  return cudaGetLastError();
}

}  // namespace sp24
