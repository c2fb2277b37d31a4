// elementwise.cu -- the bandwidth-bound kernels of the path:
//   * amax + per-tensor scale (one pass, last-block finalisation),
//   * E4M3 quantisation of activations (and the fused 6:8 lift),
//   * 2:4 magnitude prune + quantise + compress of weights,
//   * 6:8 prune + sliding-window decomposition of weights.
// All of them read 16-byte vectors with streaming loads and use grid-stride
// loops over a grid sized to the SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "quant_common.cuh"
#include "sp24.h"

namespace sp24 {

// ----------------------------------------------------------------- amax

// ws[0]: running max of |x| bits, ws[1]: finished-block ticket.  The last
// block to finish turns the max into the scale amax/448 (1.0 for amax == 0),
// flags non-finite input and re-zeroes ws.
__global__ void __launch_bounds__(256) amax_scale_kernel(const uint4 *__restrict__ x, int64_t nvec,
                                                         uint32_t *ws, float *scale_out,
                                                         int32_t *status) {
  uint32_t m = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {  // four 16-byte loads in flight
    const uint4 a = ld_stream(x + i), b = ld_stream(x + i + stride);
    const uint4 c = ld_stream(x + i + 2 * stride), d = ld_stream(x + i + 3 * stride);
    m = max(m, max(max(absmax8(a), absmax8(b)), max(absmax8(c), absmax8(d))));
  }
  for (; i < nvec; i += stride) m = max(m, absmax8(ld_stream(x + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t part[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) part[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < (blockDim.x >> 5) ? part[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) {
      atomicMax(&ws[0], m);
      __threadfence();
      const uint32_t ticket = atomicAdd(&ws[1], 1u);
      if (ticket == gridDim.x - 1) {
        __threadfence();
        const uint32_t a = atomicOr(&ws[0], 0u);
        if (a >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
        const float amax = bf16_bits_to_float(a);
        if (scale_out) *scale_out = (a == 0u) ? 1.0f : __fdiv_rn(amax, 448.0f);
        ws[0] = 0u;
        ws[1] = 0u;
        __threadfence();
      }
    }
  }
}

// ----------------------------------------------------------------- quantise

// 16 bf16 -> 16 E4M3 codes per iteration (two 16-byte loads, one store).
__global__ void __launch_bounds__(256) quantize_kernel(const uint4 *__restrict__ x, int64_t n16,
                                                       const float *__restrict__ scale,
                                                       uint4 *__restrict__ q) {
  const FastQuant qz(*scale);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride) {
    const uint4 a = ld_stream(x + 2 * i), b = ld_stream(x + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = w[2 * j], hi = w[2 * j + 1];
      o[j] = qz(lo & 0xFFFFu) | (qz(lo >> 16) << 8) | (qz(hi & 0xFFFFu) << 16) | (qz(hi >> 16) << 24);
    }
    q[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Fused quantise + 6:8 lift.  Each thread takes 16 consecutive values of a
// row (two 8-groups) and writes the 24 lifted codes
//   out[12*gl + 4*j + r] = E4M3(x[8*gl + 2*j + r] / s),  gl in {0,1}.
__global__ void __launch_bounds__(256) lift_quantize_kernel(const uint4 *__restrict__ x,
                                                            int64_t n16,
                                                            const float *__restrict__ scale,
                                                            uint2 *__restrict__ q) {
  const FastQuant qz(*scale);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride) {
    const uint4 a = ld_stream(x + 2 * i), b = ld_stream(x + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t c[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[2 * j] = qz(w[j] & 0xFFFFu);
      c[2 * j + 1] = qz(w[j] >> 16);
    }
    uint32_t out[6];
#pragma unroll
    for (int o = 0; o < 6; ++o) {
      uint32_t word = 0;
#pragma unroll
      for (int b8 = 0; b8 < 4; ++b8) {
        const int t = 4 * o + b8;  // lifted index within the 24
        const int gl = t / 12, j = (t % 12) / 4, r = t % 4;
        word |= c[8 * gl + 2 * j + r] << (8 * b8);
      }
      out[o] = word;
    }
    uint2 *dst = q + 3 * i;
    dst[0] = make_uint2(out[0], out[1]);
    dst[1] = make_uint2(out[2], out[3]);
    dst[2] = make_uint2(out[4], out[5]);
  }
}

// ----------------------------------------------------------------- 2:4 prune

// Prune/quantise/compress 8 K-values (two groups, one metadata byte).
// Codes are computed for the kept elements only, unless the pruned-dense copy
// is wanted as well.
template <bool FP8, bool DENSE>
__device__ __forceinline__ void prune8(const uint4 v, const FastQuant &qz, uint32_t kept_vals[4],
                                       uint32_t &meta_byte, uint32_t dense_out[8]) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  uint32_t h[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    h[2 * j] = words[j] & 0xFFFFu;
    h[2 * j + 1] = words[j] >> 16;
  }
  meta_byte = 0;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    uint32_t a[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) a[t] = h[4 * g + t] & 0x7FFFu;
    const uint32_t mk = keep2of4(a);
    const int i0 = __ffs(mk) - 1;
    const int i1 = __ffs(mk & (mk - 1)) - 1;
    meta_byte |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * g);
    if (DENSE) {
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t val = FP8 ? qz(h[4 * g + t]) : h[4 * g + t];
        dense_out[4 * g + t] = ((mk >> t) & 1u) ? val : 0u;
        if (t == i0) kept_vals[2 * g] = val;
        if (t == i1) kept_vals[2 * g + 1] = val;
      }
    } else {
      uint32_t h0 = 0, h1 = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (t == i0) h0 = h[4 * g + t];
        if (t == i1) h1 = h[4 * g + t];
      }
      kept_vals[2 * g] = FP8 ? qz(h0) : h0;
      kept_vals[2 * g + 1] = FP8 ? qz(h1) : h1;
    }
  }
}

// One thread per CHUNKS x 8 consecutive K-values (CHUNKS = 4 when K % 32 == 0:
// 64-byte loads, 16-byte value stores and one 4-byte metadata store).
template <bool FP8, bool DENSE, int CHUNKS>
__global__ void __launch_bounds__(256) prune24_kernel(const uint4 *__restrict__ w, int64_t nwork,
                                                      const float *__restrict__ scale,
                                                      void *__restrict__ values,
                                                      uint8_t *__restrict__ meta,
                                                      void *__restrict__ dense) {
  const FastQuant qz(FP8 ? *scale : 1.0f);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwork;
       i += stride) {
    uint4 v[CHUNKS];
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) v[c] = ld_stream(w + i * CHUNKS + c);
    uint32_t kv[CHUNKS][4], mb[CHUNKS], dn[CHUNKS][8];
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) prune8<FP8, DENSE>(v[c], qz, kv[c], mb[c], dn[c]);
    if (CHUNKS == 4) {
      reinterpret_cast<uint32_t *>(meta)[i] = mb[0] | (mb[1] << 8) | (mb[2] << 16) | (mb[3] << 24);
    } else {
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) meta[i * CHUNKS + c] = static_cast<uint8_t>(mb[c]);
    }
    if (FP8) {
      uint32_t word[CHUNKS];
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c)
        word[c] = kv[c][0] | (kv[c][1] << 8) | (kv[c][2] << 16) | (kv[c][3] << 24);
      if (CHUNKS == 4)
        reinterpret_cast<uint4 *>(values)[i] = make_uint4(word[0], word[1], word[2], word[3]);
      else
        for (int c = 0; c < CHUNKS; ++c) reinterpret_cast<uint32_t *>(values)[i * CHUNKS + c] = word[c];
      if (DENSE) {
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          uint2 d;
          d.x = dn[c][0] | (dn[c][1] << 8) | (dn[c][2] << 16) | (dn[c][3] << 24);
          d.y = dn[c][4] | (dn[c][5] << 8) | (dn[c][6] << 16) | (dn[c][7] << 24);
          reinterpret_cast<uint2 *>(dense)[i * CHUNKS + c] = d;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        reinterpret_cast<uint2 *>(values)[i * CHUNKS + c] =
            make_uint2(kv[c][0] | (kv[c][1] << 16), kv[c][2] | (kv[c][3] << 16));
        if (DENSE)
          reinterpret_cast<uint4 *>(dense)[i * CHUNKS + c] =
              make_uint4(dn[c][0] | (dn[c][1] << 16), dn[c][2] | (dn[c][3] << 16),
                         dn[c][4] | (dn[c][5] << 16), dn[c][6] | (dn[c][7] << 16));
      }
    }
  }
}

// ----------------------------------------------------------------- 6:8 decompose

// One thread per 16 K-values (two 8-groups -> 12 values, 6 nibbles = 3 bytes).
template <bool FP8>
__global__ void __launch_bounds__(256) slide68_kernel(const uint4 *__restrict__ w, int64_t n16,
                                                      const float *__restrict__ scale,
                                                      void *__restrict__ values,
                                                      uint8_t *__restrict__ meta) {
  const FastQuant qz(FP8 ? *scale : 1.0f);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride) {
    uint32_t vals[12];
    uint32_t nib[6];
#pragma unroll
    for (int gl = 0; gl < 2; ++gl) {
      const uint4 v = ld_stream(w + 2 * i + gl);
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
      uint32_t h[8], a[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        h[2 * j] = words[j] & 0xFFFFu;
        h[2 * j + 1] = words[j] >> 16;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) a[t] = h[t] & 0x7FFFu;
      int pos[6];
      assign_windows(keep6of8(a), pos);
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int p0 = pos[2 * j], p1 = pos[2 * j + 1];
        nib[3 * gl + j] = static_cast<uint32_t>((p0 - 2 * j) | ((p1 - 2 * j) << 2));
        uint32_t h0 = 0, h1 = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (t == p0) h0 = h[t];
          if (t == p1) h1 = h[t];
        }
        vals[6 * gl + 2 * j] = FP8 ? qz(h0) : h0;
        vals[6 * gl + 2 * j + 1] = FP8 ? qz(h1) : h1;
      }
    }
    uint8_t *mrow = meta + 3 * i;
    mrow[0] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
    mrow[1] = static_cast<uint8_t>(nib[2] | (nib[3] << 4));
    mrow[2] = static_cast<uint8_t>(nib[4] | (nib[5] << 4));
    if (FP8) {
      uint32_t *dst = reinterpret_cast<uint32_t *>(values) + 3 * i;
#pragma unroll
      for (int o = 0; o < 3; ++o)
        dst[o] = vals[4 * o] | (vals[4 * o + 1] << 8) | (vals[4 * o + 2] << 16) |
                 (vals[4 * o + 3] << 24);
    } else {
      uint2 *dst = reinterpret_cast<uint2 *>(values) + 3 * i;
#pragma unroll
      for (int o = 0; o < 3; ++o)
        dst[o] = make_uint2(vals[4 * o] | (vals[4 * o + 1] << 16),
                            vals[4 * o + 2] | (vals[4 * o + 3] << 16));
    }
  }
}

// ----------------------------------------------------------------- test hook
__global__ void e4m3_encode_kernel(const float *__restrict__ v, uint8_t *__restrict__ out,
                                   int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride)
    out[i] = static_cast<uint8_t>(e4m3_code(v[i]));
}

// ----------------------------------------------------------------- weight packing
// Block (t, kb) of the packed layout = 128 rows x 64 bytes of values, each
// row's 16-byte chunk c stored at position c ^ ((r >> 1) & 3) (the placement
// of the 64-byte shared-memory swizzle), then 128 rows x 16 bytes of
// metadata.  One thread per 16-byte output chunk.
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t *__restrict__ values,
                                                   const uint8_t *__restrict__ meta, int K,
                                                   int64_t nblocks, uint8_t *__restrict__ packed) {
  const int KB = K / 128;
  const int64_t nchunks = nblocks * (kPackedBlockBytes / 16);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < nchunks;
       q += stride) {
    const int64_t blk = q / (kPackedBlockBytes / 16);
    const int w = static_cast<int>(q % (kPackedBlockBytes / 16));
    const int64_t t = blk / KB;
    const int kb = static_cast<int>(blk % KB);
    const uint8_t *src;
    if (w < 512) {
      const int r = w >> 2, c = (w & 3) ^ ((r >> 1) & 3);
      src = values + (t * 128 + r) * static_cast<int64_t>(K / 2) + kb * 64 + c * 16;
    } else {
      const int r = w - 512;
      src = meta + (t * 128 + r) * static_cast<int64_t>(K / 8) + kb * 16;
    }
    reinterpret_cast<uint4 *>(packed + blk * kPackedBlockBytes)[w] = ld_stream(reinterpret_cast<const uint4 *>(src));
  }
}

// ----------------------------------------------------------------- launchers

static int grid_for(int64_t work, int sm_count) {
  const int64_t want = (work + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

cudaError_t launch_amax_scale(const void *x, int64_t nelem, uint32_t *ws, float *scale,
                              int32_t *status, int sm_count, cudaStream_t st) {
  const int64_t nvec = nelem / 8;
  amax_scale_kernel<<<grid_for(nvec, sm_count), 256, 0, st>>>(
      static_cast<const uint4 *>(x), nvec, ws, scale, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const void *x, int64_t nelem, const float *scale, uint8_t *q,
                            int sm_count, cudaStream_t st) {
  const int64_t n16 = nelem / 16;
  quantize_kernel<<<grid_for(n16, sm_count), 256, 0, st>>>(static_cast<const uint4 *>(x), n16,
                                                           scale, reinterpret_cast<uint4 *>(q));
  return cudaGetLastError();
}

cudaError_t launch_lift_quantize(const void *x, int64_t nelem, const float *scale, uint8_t *q,
                                 int sm_count, cudaStream_t st) {
  const int64_t n16 = nelem / 16;
  lift_quantize_kernel<<<grid_for(n16, sm_count), 256, 0, st>>>(
      static_cast<const uint4 *>(x), n16, scale, reinterpret_cast<uint2 *>(q));
  return cudaGetLastError();
}

template <bool FP8, bool DENSE>
static void prune24_dispatch(const void *w, int64_t nelem, bool wide, const float *scale,
                             void *values, uint8_t *meta, void *dense, int sm_count,
                             cudaStream_t st) {
  if (wide) {
    const int64_t n32 = nelem / 32;
    prune24_kernel<FP8, DENSE, 4><<<grid_for(n32, sm_count), 256, 0, st>>>(
        static_cast<const uint4 *>(w), n32, scale, values, meta, dense);
  } else {
    const int64_t n8 = nelem / 8;
    prune24_kernel<FP8, DENSE, 1><<<grid_for(n8, sm_count), 256, 0, st>>>(
        static_cast<const uint4 *>(w), n8, scale, values, meta, dense);
  }
}

cudaError_t launch_prune24(const void *w, int64_t nelem, int64_t k, bool fp8, const float *scale,
                           void *values, uint8_t *meta, void *dense, int sm_count,
                           cudaStream_t st) {
  const bool wide = k % 32 == 0;
  if (fp8) {
    if (dense) prune24_dispatch<true, true>(w, nelem, wide, scale, values, meta, dense, sm_count, st);
    else prune24_dispatch<true, false>(w, nelem, wide, scale, values, meta, dense, sm_count, st);
  } else {
    if (dense) prune24_dispatch<false, true>(w, nelem, wide, scale, values, meta, dense, sm_count, st);
    else prune24_dispatch<false, false>(w, nelem, wide, scale, values, meta, dense, sm_count, st);
  }
  return cudaGetLastError();
}

cudaError_t launch_slide68(const void *w, int64_t nelem, bool fp8, const float *scale,
                           void *values, uint8_t *meta, int sm_count, cudaStream_t st) {
  const int64_t n16 = nelem / 16;
  if (fp8)
    slide68_kernel<true><<<grid_for(n16, sm_count), 256, 0, st>>>(
        static_cast<const uint4 *>(w), n16, scale, values, meta);
  else
    slide68_kernel<false><<<grid_for(n16, sm_count), 256, 0, st>>>(
        static_cast<const uint4 *>(w), n16, scale, values, meta);
  return cudaGetLastError();
}

cudaError_t launch_pack_weights(const uint8_t *values, const uint8_t *meta, int N, int K,
                                uint8_t *packed, int sm_count, cudaStream_t st) {
  const int64_t nblocks = static_cast<int64_t>(N / 128) * (K / 128);
  pack_kernel<<<grid_for(nblocks * (kPackedBlockBytes / 16), sm_count), 256, 0, st>>>(values, meta, K,
                                                                                    nblocks, packed);
  return cudaGetLastError();
}

cudaError_t launch_e4m3_encode(const float *v, uint8_t *out, int64_t n, int sm_count,
                               cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  e4m3_encode_kernel<<<grid_for(n, sm_count), 256, 0, st>>>(v, out, n);
  return cudaGetLastError();
}

}  // namespace sp24
