// fp4.cu -- per-tensor FP4 (OCP E2M1) quantisation of activations and the
// 2:4 weight path with E2M1 codes (FP4 is among the precisions of the
// SlideSparse summary, §3 "Contribuciones Clave").
//
// The pages name the precision without a format; the rule here is the E4M3
// one on the E2M1 grid (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6): s = amax / 6
// (1.0 for an all-zero tensor), code = E2M1(RN_fp32(x / s)) rounded to the
// nearest grid value with ties to the even code, saturating at 6, the sign
// kept on a value that rounds to zero.  No block scales.  The 2:4 selection
// is that of the E4M3 path (the two largest bf16 magnitudes of each group of
// 4, ties to the lower index).
//
// Storage: two codes per byte, element 2i in the low nibble of byte i (the
// order the GEMM's 4-bit tensor-map loads read).  Activations: q [M, K/2]
// bytes.  Weights: values [N, K/2] codes = [N, K/4] bytes, metadata
// [N, K/8] in the canonical layout.
//
// Two launches, as the INT8 kernels: the CTA-reduced bf16 amax
// (amax_cta.cuh), then the encode launch, by table (a 64 KB table of the code
// of every bf16 pattern, computed for the binades that can give a nonzero
// code) or, for at most one vector per thread, by the division itself.
#include <cuda_runtime.h>
#include <stdint.h>

#include "amax_cta.cuh"
#include "fp4_kernels.h"
#include "quant_common.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kThreads = 512;
constexpr int kCtasPerSm = 2;
constexpr int kBatch = 4;          // vectors per thread per pass (table form)
constexpr int kTabBytes = 65536;   // one code per bf16 bit pattern
// |x / s| > 1/4 (the smallest value that does not round to 0) needs
// |x| > amax / 24: within 6 binades below amax's, so 7 binades in all.
constexpr int kBand = 7;

__device__ __forceinline__ uint32_t fp4_code(uint32_t h, float s) {
  return e2m1_code(__fdiv_rn(bf16_bits_to_float(h), s));
}

// FP4 code of a bf16 pattern h (16 bits): from the table, or (DIRECT) by the
// division.
template <bool DIRECT>
struct Coder {
  const uint8_t *tab;
  float s;
  __device__ __forceinline__ uint32_t operator()(uint32_t h) const {
    if constexpr (DIRECT)
      return fp4_code(h, s);
    else
      return tab[h];
  }
};

// Scale from the first launch's amax and, for the table form, this CTA's
// table: signed zeros everywhere, then the kBand binades at and below amax's
// computed by the definition.
template <bool DIRECT>
__device__ __forceinline__ Coder<DIRECT> make_coder(uint8_t *tab, const uint32_t *ws, float *scale_out,
                                                   int32_t *status) {
  __shared__ uint32_t s_amax;
  if (threadIdx.x == 0) s_amax = *reinterpret_cast<const volatile uint32_t *>(ws);
  if constexpr (!DIRECT) {
    uint4 *t4 = reinterpret_cast<uint4 *>(tab);
    for (int i = threadIdx.x; i < kTabBytes / 16; i += kThreads) {
      const uint32_t z = i < kTabBytes / 32 ? 0u : 0x08080808u;  // +0 below 0x8000, -0 above
      t4[i] = make_uint4(z, z, z, z);
    }
  }
  __syncthreads();
  const uint32_t amax = s_amax;
  const float s = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 6.0f);
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
        const uint32_t c = fp4_code(h, s);  // the code of -x is c | 8
        tab[h] = static_cast<uint8_t>(c);
        tab[h | 0x8000u] = static_cast<uint8_t>(c | 0x8u);
      }
    }
    __syncthreads();
  }
  return Coder<DIRECT>{tab, s};
}

template <bool DIRECT>
__host__ __device__ constexpr int batch() { return DIRECT ? 1 : kBatch; }

// X bf16 as nvec 16-byte vectors -> 8 codes (4 bytes) per vector.
template <bool DIRECT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    fp4_quantize_kernel(const uint4 *__restrict__ x, int64_t nvec, uint32_t *ws, float *scale_out,
                        uint32_t *__restrict__ q, int32_t *status) {
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
      uint32_t out = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) out |= (code(h[i] & 0xFFFFu) | code(h[i] >> 16) << 4) << (8 * i);
      q[v + stride * u] = out;
    }
  }
  workspace_depart(ws);
}

// W bf16 as nvec 16-byte vectors (two groups of 4; K % 8 == 0, so vector v
// owns the four kept codes 4v .. 4v + 3, i.e. value bytes 2v, 2v + 1, and
// metadata byte v of the canonical layout).
template <bool DIRECT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    fp4_prune_kernel(const uint4 *__restrict__ w, int64_t nvec, uint32_t *ws, float *scale_out,
                     uint16_t *__restrict__ values, uint8_t *__restrict__ meta, int32_t *status) {
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
        out |= (code(x0) | code(x1) << 4) << (8 * g);
      }
      values[vu] = static_cast<uint16_t>(out);
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
cudaError_t quantize_form(const uint4 *x, int64_t nvec, uint32_t *ws, float *scale, uint32_t *q, int32_t *status,
                          int sms, cudaStream_t st) {
  constexpr int smem = DIRECT ? 0 : kTabBytes;
  if constexpr (!DIRECT) {
    static const cudaError_t attr = cudaFuncSetAttribute(fp4_quantize_kernel<DIRECT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
  }
  fp4_quantize_kernel<DIRECT><<<vec_grid<DIRECT>(nvec, sms), kThreads, smem, st>>>(x, nvec, ws, scale, q, status);
  return cudaGetLastError();
}

template <bool DIRECT>
cudaError_t prune_form(const uint4 *w, int64_t nvec, uint32_t *ws, float *scale, uint16_t *values, uint8_t *meta,
                       int32_t *status, int sms, cudaStream_t st) {
  constexpr int smem = DIRECT ? 0 : kTabBytes;
  if constexpr (!DIRECT) {
    static const cudaError_t attr = cudaFuncSetAttribute(fp4_prune_kernel<DIRECT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess) return attr;
  }
  fp4_prune_kernel<DIRECT><<<vec_grid<DIRECT>(nvec, sms), kThreads, smem, st>>>(w, nvec, ws, scale, values, meta,
                                                                                status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fp4_quantize(const void *x, int64_t nelem, uint32_t *ws, float *scale, uint8_t *q,
                                int32_t *status, int sms, cudaStream_t st) {
  const int64_t nvec = nelem / 8;
  const cudaError_t e = launch_bf16_amax(x, nvec, ws, grid_cap(sms), st);
  if (e != cudaSuccess) return e;
  const uint4 *xx = static_cast<const uint4 *>(x);
  uint32_t *qq = reinterpret_cast<uint32_t *>(q);
  return direct_form(nvec, sms) ? quantize_form<true>(xx, nvec, ws, scale, qq, status, sms, st)
                                : quantize_form<false>(xx, nvec, ws, scale, qq, status, sms, st);
}

cudaError_t launch_fp4_prune24(const void *w, int64_t nelem, uint32_t *ws, float *scale, uint8_t *values,
                               uint8_t *meta, int32_t *status, int sms, cudaStream_t st) {
  const int64_t nvec = nelem / 8;
  const cudaError_t e = launch_bf16_amax(w, nvec, ws, grid_cap(sms), st);
  if (e != cudaSuccess) return e;
  const uint4 *ww = static_cast<const uint4 *>(w);
  uint16_t *vv = reinterpret_cast<uint16_t *>(values);
  return direct_form(nvec, sms) ? prune_form<true>(ww, nvec, ws, scale, vv, meta, status, sms, st)
                                : prune_form<false>(ww, nvec, ws, scale, vv, meta, status, sms, st);
}

}  // namespace sp24
