// slide.cu -- the general (2N-2):2N decomposition and lift (N = 3, 5; N = 4
// is the 6:8 path of stream.cu).
//
// SlideSparse ("SlideSparse: Fast and Flexible (2N-2):2N Structured
// Sparsity", §2 Metodologia): each 2N-group along K keeps its 2N-2 largest
// |w| (ties to the lower index) and is split into N-1 overlapping windows of
// 4 with stride 2, each exactly 2:4, over K' = K (2N-2)/N; window j of a
// group covers positions 2j .. 2j+3 and takes, in order j = 0, 1, ..., the
// two lowest-index kept positions of its range that no earlier window took.
// The activations are lifted to match: X'[m, 4((N-1)g + j) + r] =
// X[m, 2N g + 2j + r].  Both use the per-tensor E4M3 scale amax / 448.
//
// Two launches each.  The first reduces the bf16 amax into the workspace
// (one atomic per CTA).  The second derives s = amax / 448 and encodes the
// groups, in one of two forms:
//   table   (large tensors) a persistent grid of at most two CTAs per SM;
//           each fills a 64 KB table in shared memory with the E4M3 code of
//           every bf16 pattern (the 24 binades at and below amax's by the
//           definition, E4M3(RN_fp32(x / s)); signed zeros below them, where
//           x / s < 2^-13 rounds to zero) and streams the groups, a thread
//           taking a batch of four (one per 32-lane slice of its warp's span,
//           so every load instruction is coalesced) with all loads issued
//           before any is used;
//   direct  (at most one group per thread of that grid) one group per thread,
//           each code by the division itself, with no table to build.
// The last CTA to leave returns the workspace counters to zero.
#include <cuda_runtime.h>
#include <stdint.h>

#include "amax_cta.cuh"
#include "kernels.h"
#include "quant_common.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2;
constexpr int kBatch = 4;          // groups per thread per pass (table form)
constexpr int kTabBytes = 65536;   // one code per bf16 bit pattern
constexpr int kBand = 24;          // binades at and below amax's that can give a nonzero code

// The E4M3 code of a bf16 pattern h (16 bits) under the scale s: from the
// table, or (DIRECT) by the division.
template <bool DIRECT>
struct Coder {
  const uint8_t *tab;
  float s;
  __device__ __forceinline__ uint32_t operator()(uint32_t h) const {
    if constexpr (DIRECT)
      return e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s));
    else
      return tab[h];
  }
};

// Reads the amax of the first launch, publishes the scale (CTA 0) and, for
// the table form, fills this CTA's table; returns with the coder ready.
template <bool DIRECT>
__device__ __forceinline__ Coder<DIRECT> make_coder(uint8_t *tab, const uint32_t *ws, float *scale_out,
                                                   int32_t *status) {
  __shared__ uint32_t s_amax;
  if (threadIdx.x == 0) s_amax = *reinterpret_cast<const volatile uint32_t *>(ws);
  if constexpr (!DIRECT) {
    uint4 *t4 = reinterpret_cast<uint4 *>(tab);
    for (int i = threadIdx.x; i < kTabBytes / 16; i += kThreads) {
      const uint32_t z = i < kTabBytes / 32 ? 0u : 0x80808080u;  // +0 / -0 codes
      t4[i] = make_uint4(z, z, z, z);
    }
  }
  __syncthreads();
  const uint32_t amax = s_amax;
  const float s = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
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
        const uint32_t c = e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s));
        tab[h] = static_cast<uint8_t>(c);
        tab[h | 0x8000u] = static_cast<uint8_t>(c | 0x80u);
      }
    }
    __syncthreads();
  }
  return Coder<DIRECT>{tab, s};
}

// Group g of thread (warp span t, slice u): t * 32 B + 32 u + lane.
// Loads the NN words (2N bf16) of the thread's B groups, zeros past the end.
template <int NN, int B>
__device__ __forceinline__ void load_batch(const uint32_t *__restrict__ src, int64_t g0, int64_t groups,
                                           uint32_t v[B][NN]) {
#pragma unroll
  for (int u = 0; u < B; ++u) {
    const int64_t g = g0 + 32 * u;
#pragma unroll
    for (int i = 0; i < NN; ++i) v[u][i] = g < groups ? __ldg(src + g * NN + i) : 0u;
  }
}

// One 2N-group of W: drop the two smallest of the unique keys
// |w| << 4 | (15 - i) (ties to the lower index, which has the larger key),
// place the 2N-2 kept values in the N-1 windows greedily from the left, and
// write their codes (group g owns bytes 2(N-1) g of the values and N-1
// nibbles from nibble (N-1) g of the metadata).
template <int NN, class Code>
__device__ __forceinline__ void decompose_group(const uint32_t v[NN], const Code &code, int64_t g,
                                                uint8_t *__restrict__ values, uint8_t *__restrict__ meta) {
  constexpr int G2 = 2 * NN;
  uint32_t h[G2];
#pragma unroll
  for (int i = 0; i < NN; ++i) {
    h[2 * i] = v[i] & 0xFFFFu;
    h[2 * i + 1] = v[i] >> 16;
  }
  uint32_t lo1 = 0xFFFFFFFFu, lo2 = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < G2; ++i) {
    const uint32_t k = ((h[i] & 0x7FFFu) << 4) | static_cast<uint32_t>(15 - i);
    if (k < lo1) {
      lo2 = lo1;
      lo1 = k;
    } else if (k < lo2) {
      lo2 = k;
    }
  }
  uint32_t left = ((1u << G2) - 1u) & ~((1u << (15u - (lo1 & 15u))) | (1u << (15u - (lo2 & 15u))));
  uint32_t word[NN / 2] = {};
  uint32_t mbits = 0;
#pragma unroll
  for (int j = 0; j < NN - 1; ++j) {
    // slots r0 < r1 of the window (positions 2j + r); every (2N-2)-of-2N
    // mask leaves window j at least two of them
    const uint32_t cand = (left >> (2 * j)) & 0xFu;
    const int r0 = __ffs(cand) - 1;
    const int r1 = __ffs(cand & (cand - 1)) - 1;
    left &= ~(((1u << r0) | (1u << r1)) << (2 * j));
    mbits |= static_cast<uint32_t>(r0 | (r1 << 2)) << (4 * j);
    uint32_t x0 = h[2 * j], x1 = h[2 * j + 1];
#pragma unroll
    for (int r = 1; r < 4; ++r) {
      if (r == r0) x0 = h[2 * j + r];
      if (r == r1) x1 = h[2 * j + r];
    }
    word[j / 2] |= (code(x0) | code(x1) << 8) << (16 * (j & 1));
  }
  if constexpr (NN == 3) {
    *reinterpret_cast<uint32_t *>(values + g * 4) = word[0];
    meta[g] = static_cast<uint8_t>(mbits);
  } else {
    *reinterpret_cast<uint2 *>(values + g * 8) = make_uint2(word[0], word[1]);
    *reinterpret_cast<uint16_t *>(meta + g * 2) = static_cast<uint16_t>(mbits);
  }
}

// A thread's groups: B = kBatch (table form) or 1 (direct form) per warp span.
template <bool DIRECT>
__host__ __device__ constexpr int batch() { return DIRECT ? 1 : kBatch; }

template <int NN, bool DIRECT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    slide_decompose_kernel(const uint32_t *__restrict__ w, int64_t groups, uint32_t *ws, float *scale_out,
                           uint8_t *__restrict__ values, uint8_t *__restrict__ meta, int32_t *status) {
  static_assert(NN == 3 || NN == 5, "N = 3 or 5 here; 6:8 has its own kernels");
  constexpr int B = batch<DIRECT>();
  extern __shared__ __align__(16) uint8_t tab[];
  const Coder<DIRECT> code = make_coder<DIRECT>(tab, ws, scale_out, status);
  const int lane = threadIdx.x & 31;
  const int64_t span = 32 * B, warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); t * span < groups;
       t += warps) {
    uint32_t v[B][NN];
    load_batch<NN, B>(w, t * span + lane, groups, v);
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int64_t g = t * span + 32 * u + lane;
      if (g < groups) decompose_group<NN>(v[u], code, g, values, meta);
    }
  }
  workspace_depart(ws);
}

// One 2N-group of X: the 2N codes, written as the N-1 windows' 4 codes each
// (rows are whole numbers of groups, so group g's lifted bytes start at 4(N-1) g).
template <int NN, bool DIRECT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    slide_lift_kernel(const uint32_t *__restrict__ x, int64_t groups, uint32_t *ws, float *scale_out,
                      uint8_t *__restrict__ q, int32_t *status) {
  static_assert(NN == 3 || NN == 5, "N = 3 or 5 here; 6:8 has its own kernels");
  constexpr int B = batch<DIRECT>();
  extern __shared__ __align__(16) uint8_t tab[];
  const Coder<DIRECT> code = make_coder<DIRECT>(tab, ws, scale_out, status);
  const int lane = threadIdx.x & 31;
  const int64_t span = 32 * B, warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); t * span < groups;
       t += warps) {
    uint32_t v[B][NN];
    load_batch<NN, B>(x, t * span + lane, groups, v);
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int64_t g = t * span + 32 * u + lane;
      if (g >= groups) continue;
      uint32_t c[2 * NN];
#pragma unroll
      for (int i = 0; i < NN; ++i) {
        c[2 * i] = code(v[u][i] & 0xFFFFu);
        c[2 * i + 1] = code(v[u][i] >> 16);
      }
      uint32_t o[NN - 1];
#pragma unroll
      for (int j = 0; j < NN - 1; ++j) o[j] = c[2 * j] | c[2 * j + 1] << 8 | c[2 * j + 2] << 16 | c[2 * j + 3] << 24;
      if constexpr (NN == 3)
        *reinterpret_cast<uint2 *>(q + g * 8) = make_uint2(o[0], o[1]);
      else
        *reinterpret_cast<uint4 *>(q + g * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  workspace_depart(ws);
}

int64_t grid_cap(int sms) { return static_cast<int64_t>(kCtasPerSm) * sms; }

// The direct form when one group per thread fits the bounded grid.
bool direct_form(int64_t groups, int sms) { return groups <= grid_cap(sms) * kThreads; }

template <bool DIRECT>
unsigned group_grid(int64_t groups, int sms) {
  const int64_t per = static_cast<int64_t>(kThreads) * batch<DIRECT>();
  int64_t g = (groups + per - 1) / per;
  if (g > grid_cap(sms)) g = grid_cap(sms);
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

template <int NN, bool DIRECT>
cudaError_t launch_decompose_n(const uint32_t *w, int64_t groups, uint32_t *ws, float *scale, uint8_t *values,
                               uint8_t *meta, int32_t *status, int sms, cudaStream_t st) {
  constexpr int smem = DIRECT ? 0 : kTabBytes;
  if constexpr (!DIRECT) {
    // once per instantiation (thread-safe static initialisation)
    static const cudaError_t attr = cudaFuncSetAttribute(slide_decompose_kernel<NN, DIRECT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
  }
  slide_decompose_kernel<NN, DIRECT><<<group_grid<DIRECT>(groups, sms), kThreads, smem, st>>>(
      w, groups, ws, scale, values, meta, status);
  return cudaGetLastError();
}

template <int NN, bool DIRECT>
cudaError_t launch_lift_n(const uint32_t *x, int64_t groups, uint32_t *ws, float *scale, uint8_t *q,
                          int32_t *status, int sms, cudaStream_t st) {
  constexpr int smem = DIRECT ? 0 : kTabBytes;
  if constexpr (!DIRECT) {
    static const cudaError_t attr = cudaFuncSetAttribute(slide_lift_kernel<NN, DIRECT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
  }
  slide_lift_kernel<NN, DIRECT><<<group_grid<DIRECT>(groups, sms), kThreads, smem, st>>>(x, groups, ws, scale,
                                                                                        q, status);
  return cudaGetLastError();
}

template <int NN>
cudaError_t launch_decompose_form(const uint32_t *w, int64_t groups, uint32_t *ws, float *scale, uint8_t *values,
                                  uint8_t *meta, int32_t *status, int sms, cudaStream_t st) {
  return direct_form(groups, sms) ? launch_decompose_n<NN, true>(w, groups, ws, scale, values, meta, status, sms, st)
                                  : launch_decompose_n<NN, false>(w, groups, ws, scale, values, meta, status, sms, st);
}

template <int NN>
cudaError_t launch_lift_form(const uint32_t *x, int64_t groups, uint32_t *ws, float *scale, uint8_t *q,
                             int32_t *status, int sms, cudaStream_t st) {
  return direct_form(groups, sms) ? launch_lift_n<NN, true>(x, groups, ws, scale, q, status, sms, st)
                                  : launch_lift_n<NN, false>(x, groups, ws, scale, q, status, sms, st);
}

}  // namespace

cudaError_t launch_slide_decompose(const void *w, int N, int K, int n, uint32_t *ws, float *scale,
                                   uint8_t *values, uint8_t *meta, int32_t *status, int sms, cudaStream_t st) {
  if (n != 3 && n != 5) return cudaErrorInvalidValue;
  const cudaError_t e = launch_bf16_amax(w, static_cast<int64_t>(N) * K / 8, ws, grid_cap(sms), st);
  if (e != cudaSuccess) return e;
  const int64_t groups = static_cast<int64_t>(N) * (K / (2 * n));
  const uint32_t *ww = static_cast<const uint32_t *>(w);
  return n == 3 ? launch_decompose_form<3>(ww, groups, ws, scale, values, meta, status, sms, st)
                : launch_decompose_form<5>(ww, groups, ws, scale, values, meta, status, sms, st);
}

cudaError_t launch_slide_lift(const void *x, int M, int K, int n, uint32_t *ws, float *scale, uint8_t *q,
                              int32_t *status, int sms, cudaStream_t st) {
  if (n != 3 && n != 5) return cudaErrorInvalidValue;
  const cudaError_t e = launch_bf16_amax(x, static_cast<int64_t>(M) * K / 8, ws, grid_cap(sms), st);
  if (e != cudaSuccess) return e;
  const int64_t groups = static_cast<int64_t>(M) * (K / (2 * n));
  const uint32_t *xx = static_cast<const uint32_t *>(x);
  return n == 3 ? launch_lift_form<3>(xx, groups, ws, scale, q, status, sms, st)
                : launch_lift_form<5>(xx, groups, ws, scale, q, status, sms, st);
}

}  // namespace sp24
