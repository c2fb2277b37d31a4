// int8.cu -- symmetric per-tensor INT8 quantisation of activations and the
// 2:4 weight path with INT8 codes (the W8A8 recipe of the cookbook's
// Comparison Tables; INT8 is among the precisions of the SlideSparse summary,
// §3 "Contribuciones Clave").
//
// The pages name the recipe without a formula; the rule here is the E4M3 one
// on the INT8 grid: s = amax / 127 (1.0 for an all-zero tensor) and
// q = clamp(round_half_even(RN_fp32(x / s)), -127, 127).  The 2:4 selection is
// that of the E4M3 path (the two largest bf16 magnitudes of each group of 4,
// ties to the lower index), written in the canonical layout: values int8
// [N, K/2], metadata [N, K/8].
//
// Two launches, as the general sliding-window kernels: the CTA-reduced bf16
// amax (amax_cta.cuh), then the encode launch in one of two forms --
//   table   a persistent grid of at most two CTAs per SM, each filling a
//           64 KB table with the code of every bf16 pattern (computed for the
//           10 binades at and below amax's; below them |x / s| < 0.5, code 0)
//           and streaming 16-byte vectors, four per thread per pass;
//   direct  at most one vector per thread of that grid: the division itself.
// The last CTA of the encode launch returns the workspace counters to zero.
#include <cuda_runtime.h>
#include <stdint.h>

#include "amax_cta.cuh"
#include "int8_kernels.h"
#include "quant_common.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2;
constexpr int kBatch = 4;          // vectors per thread per pass (table form)
constexpr int kTabBytes = 65536;   // one code per bf16 bit pattern
constexpr int kBand = 10;          // |x| >= amax / 254 lies within 9 binades of amax's

// INT8 code (as its byte) of a bf16 pattern h (16 bits): from the table, or
// (DIRECT) by the division.
template <bool DIRECT>
struct Coder {
  const uint8_t *tab;
  float s;
  __device__ __forceinline__ uint32_t operator()(uint32_t h) const {
    if constexpr (DIRECT)
      return static_cast<uint32_t>(int8_code(h, s)) & 0xFFu;
    else
      return tab[h];
  }
};

// Scale from the first launch's amax (CTA 0 publishes it) and, for the table
// form, this CTA's table; returns with the coder ready.
template <bool DIRECT>
__device__ __forceinline__ Coder<DIRECT> make_coder(uint8_t *tab, const uint32_t *ws, float *scale_out,
                                                   int32_t *status) {
  __shared__ uint32_t s_amax;
  if (threadIdx.x == 0) s_amax = *reinterpret_cast<const volatile uint32_t *>(ws);
  if constexpr (!DIRECT) {
    uint4 *t4 = reinterpret_cast<uint4 *>(tab);
    for (int i = threadIdx.x; i < kTabBytes / 16; i += kThreads) t4[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  const uint32_t amax = s_amax;
  const float s = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 127.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (scale_out) *scale_out = s;
    if (amax >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
  }
  if constexpr (!DIRECT) {
    const int e0 = static_cast<int>(amax >> 7) - (kBand - 1);
    for (int i = threadIdx.x; i < kBand * 128; i += kThreads) {
      const int e = e0 + (i >> 7);
      if (e >= 0 && e < 255) {
        const uint32_t h = static_cast<uint32_t>(e) << 7 | static_cast<uint32_t>(i & 127);
        const int32_t c = int8_code(h, s);  // the code of -x is -c
        tab[h] = static_cast<uint8_t>(c);
        tab[h | 0x8000u] = static_cast<uint8_t>(-c);
      }
    }
    __syncthreads();
  }
  return Coder<DIRECT>{tab, s};
}

template <bool DIRECT>
__host__ __device__ constexpr int batch() { return DIRECT ? 1 : kBatch; }

// X bf16 as nvec 16-byte vectors -> 8 codes per vector.
template <bool DIRECT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    int8_quantize_kernel(const uint4 *__restrict__ x, int64_t nvec, uint32_t *ws, float *scale_out,
                         uint2 *__restrict__ q, int32_t *status) {
  constexpr int B = batch<DIRECT>();
  extern __shared__ __align__(16) uint8_t tab[];
  const Coder<DIRECT> code = make_coder<DIRECT>(tab, ws, scale_out, status);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; v < nvec; v += stride * B) {
    uint4 w[B];
#pragma unroll
    for (int u = 0; u < B; ++u) w[u] = v + stride * u < nvec ? __ldg(x + v + stride * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < B; ++u) {
      if (v + stride * u >= nvec) break;
      const uint32_t h[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        lo |= (code(h[i] & 0xFFFFu) | code(h[i] >> 16) << 8) << (16 * i);
        hi |= (code(h[2 + i] & 0xFFFFu) | code(h[2 + i] >> 16) << 8) << (16 * i);
      }
      q[v + stride * u] = make_uint2(lo, hi);
    }
  }
  workspace_depart(ws);
}

// W bf16 as nvec 16-byte vectors (two groups of 4 each; K % 8 == 0, so a
// vector never straddles rows and vector v owns value bytes 4v .. 4v + 3 and
// metadata byte v of the canonical layout).
template <bool DIRECT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    int8_prune_kernel(const uint4 *__restrict__ w, int64_t nvec, uint32_t *ws, float *scale_out,
                      uint32_t *__restrict__ values, uint8_t *__restrict__ meta, int32_t *status) {
  constexpr int B = batch<DIRECT>();
  extern __shared__ __align__(16) uint8_t tab[];
  const Coder<DIRECT> code = make_coder<DIRECT>(tab, ws, scale_out, status);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; v < nvec; v += stride * B) {
    uint4 wv[B];
#pragma unroll
    for (int u = 0; u < B; ++u)
      wv[u] = v + stride * u < nvec ? __ldg(w + v + stride * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int64_t vu = v + stride * u;
      if (vu >= nvec) break;
      const uint32_t h[8] = {wv[u].x & 0xFFFFu, wv[u].x >> 16, wv[u].y & 0xFFFFu, wv[u].y >> 16,
                             wv[u].z & 0xFFFFu, wv[u].z >> 16, wv[u].w & 0xFFFFu, wv[u].w >> 16};
      uint32_t out = 0, mb = 0;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t a[4] = {h[4 * g] & 0x7FFFu, h[4 * g + 1] & 0x7FFFu, h[4 * g + 2] & 0x7FFFu,
                               h[4 * g + 3] & 0x7FFFu};
        const uint32_t keep = keep2of4(a);
        const int i0 = __ffs(keep) - 1, i1 = __ffs(keep & (keep - 1)) - 1;
        uint32_t x0 = h[4 * g], x1 = h[4 * g + 1];
#pragma unroll
        for (int r = 1; r < 4; ++r) {
          if (r == i0) x0 = h[4 * g + r];
          if (r == i1) x1 = h[4 * g + r];
        }
        mb |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * g);
        out |= (code(x0) | code(x1) << 8) << (16 * g);
      }
      values[vu] = out;
      meta[vu] = static_cast<uint8_t>(mb);
    }
  }
  workspace_depart(ws);
}

int64_t grid_cap(int sms) { return static_cast<int64_t>(kCtasPerSm) * sms; }

// The direct form when one vector per thread fits the bounded grid.
bool direct_form(int64_t nvec, int sms) { return nvec <= grid_cap(sms) * kThreads; }

template <bool DIRECT>
unsigned vec_grid(int64_t nvec, int sms) {
  const int64_t per = static_cast<int64_t>(kThreads) * batch<DIRECT>();
  int64_t g = (nvec + per - 1) / per;
  if (g > grid_cap(sms)) g = grid_cap(sms);
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

template <bool DIRECT>
cudaError_t quantize_form(const uint4 *x, int64_t nvec, uint32_t *ws, float *scale, uint2 *q, int32_t *status,
                          int sms, cudaStream_t st) {
  constexpr int smem = DIRECT ? 0 : kTabBytes;
  if constexpr (!DIRECT) {
    // once per instantiation (thread-safe static initialisation)
    static const cudaError_t attr = cudaFuncSetAttribute(int8_quantize_kernel<DIRECT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
  }
  int8_quantize_kernel<DIRECT><<<vec_grid<DIRECT>(nvec, sms), kThreads, smem, st>>>(x, nvec, ws, scale, q, status);
  return cudaGetLastError();
}

template <bool DIRECT>
cudaError_t prune_form(const uint4 *w, int64_t nvec, uint32_t *ws, float *scale, uint32_t *values, uint8_t *meta,
                       int32_t *status, int sms, cudaStream_t st) {
  constexpr int smem = DIRECT ? 0 : kTabBytes;
  if constexpr (!DIRECT) {
    static const cudaError_t attr = cudaFuncSetAttribute(int8_prune_kernel<DIRECT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
  }
  int8_prune_kernel<DIRECT><<<vec_grid<DIRECT>(nvec, sms), kThreads, smem, st>>>(w, nvec, ws, scale, values, meta,
                                                                                 status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_int8_quantize(const void *x, int64_t nelem, uint32_t *ws, float *scale, int8_t *q,
                                 int32_t *status, int sms, cudaStream_t st) {
  const int64_t nvec = nelem / 8;
  const cudaError_t e = launch_bf16_amax(x, nvec, ws, grid_cap(sms), st);
  if (e != cudaSuccess) return e;
  const uint4 *xx = static_cast<const uint4 *>(x);
  uint2 *qq = reinterpret_cast<uint2 *>(q);
  return direct_form(nvec, sms) ? quantize_form<true>(xx, nvec, ws, scale, qq, status, sms, st)
                                : quantize_form<false>(xx, nvec, ws, scale, qq, status, sms, st);
}

cudaError_t launch_int8_prune24(const void *w, int64_t nelem, uint32_t *ws, float *scale, int8_t *values,
                                uint8_t *meta, int32_t *status, int sms, cudaStream_t st) {
  const int64_t nvec = nelem / 8;
  const cudaError_t e = launch_bf16_amax(w, nvec, ws, grid_cap(sms), st);
  if (e != cudaSuccess) return e;
  const uint4 *ww = static_cast<const uint4 *>(w);
  uint32_t *vv = reinterpret_cast<uint32_t *>(values);
  return direct_form(nvec, sms) ? prune_form<true>(ww, nvec, ws, scale, vv, meta, status, sms, st)
                                : prune_form<false>(ww, nvec, ws, scale, vv, meta, status, sms, st);
}

}  // namespace sp24
