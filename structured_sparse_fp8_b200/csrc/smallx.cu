// smallx.cu -- per-tensor quantisation of decode-sized activations by ONE
// thread-block cluster: E4M3 codes, the SlideSparse 6:8 lift of them, INT8
// codes or FP4 (E2M1) codes.
//
// The quantiser of the cookbook's FP8 recipe ("Practical Example 2": one
// scale amax / 448 for the whole tensor, codes E4M3(x / scale)) needs the
// amax of all of X before the first code.  For a decode batch (X of at most
// kSmallXVec 16-byte vectors, 256 KB of bf16) a grid-wide two-phase kernel is
// all latency: its grid barrier alone costs microseconds while HBM streams
// the GEMM's weights.  Here a single cluster of kSmallCtas CTAs does it with
// no global synchronisation at all:
//  1. CTA r loads its slice of X (contiguous 8-element vectors) into
//     registers, at most kSmallRegs vectors per thread, all loads in flight;
//  2. reduces the slice to its largest |x| bit pattern, stores it in slot r
//     of every CTA of the cluster (distributed shared memory) and arrives on
//     each one's mbarrier (release, cluster scope);
//  3. waits for its own barrier's kSmallCtas arrivals (acquire, cluster
//     scope), takes the max of the slots and the scale s = amax / 448
//     (1 when amax = 0);
//  4. encodes its registers and stores them: E4M3 with the division-free
//     encoder (e4m3_codes8_fast, exact; the vectors it cannot decide go
//     through the correctly rounded division), 8 codes or the 12 lifted
//     codes per vector; INT8 (s = amax / 127) and FP4 (s = amax / 6) by the
//     correctly rounded division, 8 bytes or 8 nibbles (element 2i in the
//     low nibble of byte i) per vector.
// The kernel releases its dependents as soon as the previous kernel has
// completed: the GEMM that consumes the codes then launches and streams its
// weights while this cluster runs (it waits for this grid's completion
// before reading codes or scale).  Released at entry instead, that GEMM
// competed with the kernel before this one and the chain was slower.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "quant_common.cuh"
#include "sm100_ptx.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kSmallCtas = 8;    // one portable-size cluster
constexpr int kSmallThreads = 256;
constexpr int kSmallRegs = 8;    // 16-byte X vectors per thread

// amax / (the code grid's largest magnitude) is the scale
__host__ __device__ constexpr float grid_max(int enc) {
  return enc == kSmallInt8 ? 127.0f : enc == kSmallFp4 ? 6.0f : 448.0f;
}

template <int ENC>
__global__ void __launch_bounds__(kSmallThreads)
    small_quantize_kernel(const uint4 *__restrict__ x, int64_t nvec, float *scale_out, uint8_t *__restrict__ q,
                          int32_t *status) {
  __shared__ uint64_t bar;
  __shared__ uint32_t s_part[kSmallCtas];
  __shared__ uint32_t s_red[kSmallThreads / 32];
  __shared__ float s_scale[2];
  const int t = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  if (t == 0) {
    mbar_init(&bar, kSmallCtas);
    fence_mbar_init();
  }
  cluster_sync_all();  // every CTA's barrier is initialised before any remote arrive
  grid_dependency_wait();  // X may come from the previous kernel
  grid_launch_dependents();

  const int64_t v0 = static_cast<int64_t>(rank) * nvec / kSmallCtas;
  const int64_t v1 = static_cast<int64_t>(rank + 1) * nvec / kSmallCtas;
  uint4 w[kSmallRegs];
#pragma unroll
  for (int u = 0; u < kSmallRegs; ++u) {
    const int64_t v = v0 + t + kSmallThreads * u;
    w[u] = v < v1 ? __ldg(x + v) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t m2 = 0;
#pragma unroll
  for (int u = 0; u < kSmallRegs; ++u) m2 = __vmaxu2(m2, absmax8x2(w[u]));
  const uint32_t mw = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
  if ((t & 31) == 0) s_red[t >> 5] = mw;
  __syncthreads();
  if (t < kSmallCtas) {
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kSmallThreads / 32; ++i) mx = max(mx, s_red[i]);
    st_shared_cluster(mapa_shared(&s_part[rank], t), mx);
    mbar_arrive_cluster(mapa_shared(&bar, t));
  }
  if (t == 0) {
    mbar_wait_cluster(&bar, 0u, status);
    uint32_t amax = 0;
#pragma unroll
    for (int r = 0; r < kSmallCtas; ++r) amax = max(amax, s_part[r]);
    const float sx = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), grid_max(ENC));
    if (rank == 0) {
      *scale_out = sx;
      if (amax >= 0x7F80u && status) atomicOr(status, SP24_STATUS_NONFINITE);
    }
    s_scale[0] = sx;
    s_scale[1] = __frcp_rn(sx);
  }
  __syncthreads();
  const float sx = s_scale[0], rx = s_scale[1];
  if constexpr (ENC == kSmallInt8 || ENC == kSmallFp4) {
#pragma unroll
    for (int u = 0; u < kSmallRegs; ++u) {
      const int64_t v = v0 + t + kSmallThreads * u;
      if (v < v1) {
        const uint32_t h[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t e = (h[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
          if constexpr (ENC == kSmallInt8) {
            const uint32_t b = static_cast<uint32_t>(int8_code(e, sx)) & 0xFFu;
            if (i < 4) lo |= b << (8 * i); else hi |= b << (8 * (i - 4));
          } else {
            lo |= e2m1_code(__fdiv_rn(bf16_bits_to_float(e), sx)) << (4 * i);
          }
        }
        if constexpr (ENC == kSmallInt8)
          *reinterpret_cast<uint2 *>(q + 8 * v) = make_uint2(lo, hi);
        else
          *reinterpret_cast<uint32_t *>(q + 4 * v) = lo;
      }
    }
  } else {
    uint2 c[kSmallRegs];
    bool ok[kSmallRegs];
#pragma unroll
    for (int u = 0; u < kSmallRegs; ++u) c[u] = e4m3_codes8_fast(w[u], rx, ok[u]);
#pragma unroll
    for (int u = 0; u < kSmallRegs; ++u) {
      const int64_t v = v0 + t + kSmallThreads * u;
      if (v < v1) {
        if (!ok[u]) c[u] = e4m3_codes8_div(w[u], sx);
        if constexpr (ENC == kSmallLift) {
          // 8-group g -> the 12 codes of windows 2j .. 2j + 3, j = 0..2
          uint32_t *o = reinterpret_cast<uint32_t *>(q + 12 * v);
          o[0] = c[u].x;
          o[1] = __byte_perm(c[u].x, c[u].y, 0x5432);
          o[2] = c[u].y;
        } else {
          *reinterpret_cast<uint2 *>(q + 8 * v) = c[u];
        }
      }
    }
  }
  // No CTA leaves while a peer may still write to its shared memory (only
  // possible after a wait above timed out).
  cluster_sync_all();
}

}  // namespace

bool small_quantize_fits(int64_t nelem) { return nelem > 0 && nelem % 8 == 0 && nelem / 8 <= kSmallXVec; }

cudaError_t launch_quantize_small(const void *x, int64_t nelem, SmallEnc enc, float *scale, uint8_t *q,
                                  int32_t *status, cudaStream_t st) {
  static_assert(kSmallXVec <= static_cast<int64_t>(kSmallCtas) * kSmallThreads * kSmallRegs,
                "every vector of a small X is held in some thread's registers");
  if (!small_quantize_fits(nelem)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSmallCtas, 1, 1);
  cfg.blockDim = dim3(kSmallThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  attrs[1].id = cudaLaunchAttributeClusterDimension;
  attrs[1].val.clusterDim.x = kSmallCtas;
  attrs[1].val.clusterDim.y = 1;
  attrs[1].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  const uint4 *xv = static_cast<const uint4 *>(x);
  const int64_t nvec = nelem / 8;
  switch (enc) {
    case kSmallE4M3: return cudaLaunchKernelEx(&cfg, small_quantize_kernel<kSmallE4M3>, xv, nvec, scale, q, status);
    case kSmallLift: return cudaLaunchKernelEx(&cfg, small_quantize_kernel<kSmallLift>, xv, nvec, scale, q, status);
    case kSmallInt8: return cudaLaunchKernelEx(&cfg, small_quantize_kernel<kSmallInt8>, xv, nvec, scale, q, status);
    case kSmallFp4: return cudaLaunchKernelEx(&cfg, small_quantize_kernel<kSmallFp4>, xv, nvec, scale, q, status);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sp24
