// stream.cu -- the bandwidth-bound steps of the path as single-launch,
// TMA-streamed kernels:
//   kOpQuantize  per-tensor E4M3 quantisation of activations,
//   kOpLift      the same fused with the 6:8 activation lift,
//   kOpPrune24   2:4 magnitude prune + quantise + compress of weights,
//   kOpSlide68   6:8 prune + sliding-window decomposition of weights.
//
// One CTA per SM (cooperative launch: all CTAs resident), each owning a
// contiguous range of 32 KB chunks of the bf16 input.  A producer warp
// streams the chunks into a 6-stage shared-memory ring with bulk TMA copies
// (full/empty mbarriers per slot), 16 consumer warps work on interleaved
// 16-byte units of each chunk.
//   Phase 1: amax of the slice (and, for the prune ops, the group selection,
//            whose metadata is written straight to global memory).
//   Grid barrier: the CTAs combine their amax through device counters that
//            the last CTA to leave resets; every CTA derives s = amax / 448
//            and fills a 3 KB code table in shared memory with the E4M3 code
//            of every bf16 magnitude that can produce a nonzero code (the 24
//            binades below amax), each entry computed as the definition
//            states: E4M3(RN_fp32(x / s)).
//   Phase 2: codes by table lookup; the slice comes from the ring again when
//            the CTA's whole range fitted in it, else it is re-streamed
//            (normally from L2).
// The bf16-output prune ops need no scale and finish after phase 1.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"
#include "quant_common.cuh"
#include "sm100_ptx.cuh"
#include "sp24.h"

namespace sp24 {

namespace {

constexpr int kConsumers = 512;              // 16 consumer warps
constexpr int kThreads = kConsumers + 32;    // + one producer warp
constexpr int kChunkBytes = 32768;
constexpr int kStages = 6;
constexpr int kTab = 24 * 128;               // 24 binades x 128 mantissas
constexpr uint32_t kSmemBytes = kStages * kChunkBytes + kTab + 2 * kStages * 8 + 128;

enum StreamOp : int { kOpQuantize = 0, kOpLift = 1, kOpPrune24 = 2, kOpSlide68 = 3 };

// Bytes of input one consumer thread handles as one unit: 8 bf16 (one
// metadata byte of 2:4, one 8-group of the lift) or 16 bf16 for 6:8 (two
// 8-groups = three metadata bytes).  Unit r of thread t in a chunk starts at
// byte r * kConsumers * kUnit + t * kUnit: consecutive threads read
// consecutive 16-byte words (no shared-memory bank conflicts) and write
// consecutive outputs.
template <int OP>
__host__ __device__ constexpr int unit_bytes() { return OP == kOpSlide68 ? 32 : 16; }

struct StreamArgs {
  const uint8_t *x;  // bf16 input
  int64_t nbytes;    // input bytes, a multiple of 32
  int64_t nchunks;
  uint32_t *ws;      // [0] amax bits, [1] arrivals, [2] departures
  float *scale_out;
  int32_t *status;
  uint8_t *out;      // codes / kept values
  uint8_t *meta;
  uint8_t *dense;
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// E4M3 code of a bf16 pattern by lookup: entry i of the table holds the
// magnitude code of exponent field (base7 >> 7) + i / 128, mantissa i % 128.
// Smaller magnitudes are below 2^-13 after division and encode to +-0.
// With `direct` set (tensors too small to amortise the table) the code is
// computed by the same division directly.
struct CodeTable {
  const uint8_t *tab;
  int base7;
  float s;
  bool direct;
  __device__ __forceinline__ uint32_t operator()(uint32_t h) const {
    if (direct) return e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s));
    const int idx = static_cast<int>(h & 0x7FFFu) - base7;
    const uint32_t c = static_cast<unsigned>(idx) < static_cast<unsigned>(kTab) ? tab[idx] : 0u;
    return c | ((h >> 8) & 0x80u);
  }
};

__device__ __forceinline__ void build_table(uint8_t *tab, uint32_t amax_bits, float s, int t) {
  const int e_base = static_cast<int>(amax_bits >> 7) - 23;
  for (int i = t; i < kTab; i += kConsumers) {
    const int e = e_base + i / 128;
    uint32_t c = 0;
    if (e >= 0 && e < 255) {
      const uint32_t h = (static_cast<uint32_t>(e) << 7) | static_cast<uint32_t>(i & 127);
      c = e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s)) & 0x7Fu;
    }
    tab[i] = static_cast<uint8_t>(c);
  }
}

__device__ __forceinline__ void halves(const uint4 v, uint32_t h[8]) {
  h[0] = v.x & 0xFFFFu; h[1] = v.x >> 16; h[2] = v.y & 0xFFFFu; h[3] = v.y >> 16;
  h[4] = v.z & 0xFFFFu; h[5] = v.z >> 16; h[6] = v.w & 0xFFFFu; h[7] = v.w >> 16;
}

// ------------------------------------------------------------------ phase 1
// One unit: `p` its bytes in shared memory, `e0` the index of its first element.
template <int OP, bool FP8, bool DENSE>
__device__ __forceinline__ uint32_t phase1_unit(const uint8_t *p, int64_t e0, const StreamArgs &a) {
  if constexpr (OP == kOpSlide68) {
    const uint4 v0 = reinterpret_cast<const uint4 *>(p)[0];
    const uint4 v1 = reinterpret_cast<const uint4 *>(p)[1];
    uint32_t nib[6], vals[12];
#pragma unroll
    for (int gl = 0; gl < 2; ++gl) {
      uint32_t h[8], aa[8];
      halves(gl ? v1 : v0, h);
#pragma unroll
      for (int t = 0; t < 8; ++t) aa[t] = h[t] & 0x7FFFu;
      int pos[6];
      assign_windows(keep6of8(aa), pos);
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int p0 = pos[2 * j], p1 = pos[2 * j + 1];
        nib[3 * gl + j] = static_cast<uint32_t>((p0 - 2 * j) | ((p1 - 2 * j) << 2));
        if (!FP8) {
          uint32_t h0 = 0, h1 = 0;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (t == p0) h0 = h[t];
            if (t == p1) h1 = h[t];
          }
          vals[6 * gl + 2 * j] = h0;
          vals[6 * gl + 2 * j + 1] = h1;
        }
      }
    }
    const int64_t unit = e0 / 16;
    uint8_t *m = a.meta + 3 * unit;
    m[0] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
    m[1] = static_cast<uint8_t>(nib[2] | (nib[3] << 4));
    m[2] = static_cast<uint8_t>(nib[4] | (nib[5] << 4));
    if (!FP8) {
      uint2 *d = reinterpret_cast<uint2 *>(a.out + 24 * unit);
#pragma unroll
      for (int o = 0; o < 3; ++o)
        d[o] = make_uint2(vals[4 * o] | (vals[4 * o + 1] << 16), vals[4 * o + 2] | (vals[4 * o + 3] << 16));
    }
    return max(absmax8(v0), absmax8(v1));
  } else {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    if constexpr (OP == kOpPrune24) {
      uint32_t h[8];
      halves(v, h);
      uint32_t mb = 0, kept[4], dn[8];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t aa[4] = {h[4 * g] & 0x7FFFu, h[4 * g + 1] & 0x7FFFu, h[4 * g + 2] & 0x7FFFu,
                                h[4 * g + 3] & 0x7FFFu};
        const uint32_t mk = keep2of4(aa);
        const int i0 = __ffs(mk) - 1, i1 = __ffs(mk & (mk - 1)) - 1;
        mb |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * g);
        if (!FP8) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (t == i0) kept[2 * g] = h[4 * g + t];
            if (t == i1) kept[2 * g + 1] = h[4 * g + t];
            if (DENSE) dn[4 * g + t] = ((mk >> t) & 1u) ? h[4 * g + t] : 0u;
          }
        }
      }
      a.meta[e0 / 8] = static_cast<uint8_t>(mb);
      if (!FP8) {
        *reinterpret_cast<uint2 *>(a.out + e0) =
            make_uint2(kept[0] | (kept[1] << 16), kept[2] | (kept[3] << 16));
        if (DENSE)
          *reinterpret_cast<uint4 *>(a.dense + 2 * e0) =
              make_uint4(dn[0] | (dn[1] << 16), dn[2] | (dn[3] << 16), dn[4] | (dn[5] << 16),
                         dn[6] | (dn[7] << 16));
      }
    }
    return absmax8(v);
  }
}

// ------------------------------------------------------------------ phase 2
// `meta_in` is the unit's metadata (one byte for 2:4, three for 6:8), loaded
// before the chunk's stores so that the loads overlap.
template <int OP, bool DENSE>
__device__ __forceinline__ void phase2_unit(const uint8_t *p, int64_t e0, uint32_t meta_in,
                                            const StreamArgs &a, const CodeTable &code) {
  if constexpr (OP == kOpSlide68) {
    const uint4 v0 = reinterpret_cast<const uint4 *>(p)[0];
    const uint4 v1 = reinterpret_cast<const uint4 *>(p)[1];
    const int64_t unit = e0 / 16;
    const uint32_t m3 = meta_in;
    uint32_t c[12];
#pragma unroll
    for (int gl = 0; gl < 2; ++gl) {
      uint32_t h[8];
      halves(gl ? v1 : v0, h);
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const uint32_t nib = (m3 >> (4 * (3 * gl + j))) & 0xFu;
        const uint32_t p0 = 2 * j + (nib & 3u), p1 = 2 * j + (nib >> 2);
        uint32_t h0 = 0, h1 = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (p0 == static_cast<uint32_t>(t)) h0 = h[t];
          if (p1 == static_cast<uint32_t>(t)) h1 = h[t];
        }
        c[6 * gl + 2 * j] = code(h0);
        c[6 * gl + 2 * j + 1] = code(h1);
      }
    }
    uint32_t *d = reinterpret_cast<uint32_t *>(a.out + 12 * unit);
#pragma unroll
    for (int o = 0; o < 3; ++o)
      d[o] = c[4 * o] | (c[4 * o + 1] << 8) | (c[4 * o + 2] << 16) | (c[4 * o + 3] << 24);
  } else {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    uint32_t h[8];
    halves(v, h);
    if constexpr (OP == kOpQuantize) {
      *reinterpret_cast<uint2 *>(a.out + e0) =
          make_uint2(code(h[0]) | (code(h[1]) << 8) | (code(h[2]) << 16) | (code(h[3]) << 24),
                     code(h[4]) | (code(h[5]) << 8) | (code(h[6]) << 16) | (code(h[7]) << 24));
    } else if constexpr (OP == kOpLift) {
      // lifted[12 g + 4 j + r] = code(x[8 g + 2 j + r]) for the 8-group g
      uint32_t c[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) c[t] = code(h[t]);
      uint32_t *d = reinterpret_cast<uint32_t *>(a.out + 12 * (e0 / 8));
      d[0] = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
      d[1] = c[2] | (c[3] << 8) | (c[4] << 16) | (c[5] << 24);
      d[2] = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
    } else if constexpr (OP == kOpPrune24) {
      const uint32_t mb = meta_in;
      uint32_t c[4], dn[2];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t nib = (mb >> (4 * g)) & 0xFu;
        const uint32_t i0 = nib & 3u, i1 = nib >> 2;
        uint32_t h0 = h[4 * g], h1 = h[4 * g + 1];
#pragma unroll
        for (int t = 1; t < 4; ++t) {
          if (i0 == static_cast<uint32_t>(t)) h0 = h[4 * g + t];
          if (i1 == static_cast<uint32_t>(t)) h1 = h[4 * g + t];
        }
        c[2 * g] = code(h0);
        c[2 * g + 1] = code(h1);
        if (DENSE) dn[g] = (c[2 * g] << (8 * i0)) | (c[2 * g + 1] << (8 * i1));
      }
      *reinterpret_cast<uint32_t *>(a.out + e0 / 2) = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
      if (DENSE) *reinterpret_cast<uint2 *>(a.dense + e0) = make_uint2(dn[0], dn[1]);
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int OP, bool FP8, bool DENSE>
__global__ void __launch_bounds__(kThreads, 1) stream_kernel(const StreamArgs a) {
  constexpr int kUnit = unit_bytes<OP>();
  constexpr int kRows = kChunkBytes / (kConsumers * kUnit);  // units per thread per chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  uint8_t *tab = ring + kStages * kChunkBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(tab + kTab);
  uint64_t *empty = full + kStages;
  __shared__ uint32_t s_red[kConsumers / 32];
  __shared__ uint32_t s_amax;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * a.nchunks / gridDim.x;
  const int64_t c1 = static_cast<int64_t>(blockIdx.x + 1) * a.nchunks / gridDim.x;
  const int n_my = static_cast<int>(c1 - c0);
  const bool resident = n_my <= kStages;             // phase 2 reuses the ring contents
  const int n_loads = (FP8 && !resident) ? 2 * n_my : n_my;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_wait();
  // Activation kernels let the next kernel (a GEMM) launch early; the weight
  // path never does, which is what allows a GEMM to prefetch weights before
  // its own dependency wait.
  if (OP == kOpQuantize || OP == kOpLift) grid_launch_dependents();

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    // Load L brings chunk c0 + L % n_my into slot L % kStages.  The second
    // pass over the chunks (phase 2) is prefetched as soon as slots free up.
    if ((tid & 31) == 0) {
      for (int L = 0; L < n_loads; ++L) {
        const int slot = L % kStages;
        if (L >= kStages &&
            !mbar_wait(&empty[slot], static_cast<uint32_t>(L / kStages - 1) & 1u, a.status))
          break;
        const int64_t c = c0 + L % n_my;
        const uint32_t nb =
            static_cast<uint32_t>(min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes));
        mbar_arrive_expect_tx(&full[slot], nb);
        bulk_load(ring + slot * kChunkBytes, a.x + c * kChunkBytes, nb, &full[slot]);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  auto for_units = [&](const uint8_t *chunk, int64_t c, auto &&fn) {
    const int64_t nb = min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int off = (r * kConsumers + tid) * kUnit;
      if (off < nb) fn(chunk + off, (c * kChunkBytes + off) / 2);
    }
  };

  uint32_t mx = 0;
  for (int i = 0; i < n_my; ++i) {
    const int slot = i % kStages;
    mbar_wait(&full[slot], static_cast<uint32_t>(i / kStages) & 1u, a.status);
    for_units(ring + slot * kChunkBytes, c0 + i, [&](const uint8_t *p, int64_t e0) {
      mx = max(mx, phase1_unit<OP, FP8, DENSE>(p, e0, a));
    });
    __syncwarp();
    if (!resident && (tid & 31) == 0) mbar_arrive(&empty[slot]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if ((tid & 31) == 0) s_red[warp] = mx;
  named_bar_sync(1, kConsumers);
  if (tid < 32) {
    mx = tid < kConsumers / 32 ? s_red[tid] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  }

  if constexpr (!FP8) {
    // bf16 outputs are complete; only the finiteness check remains
    if (tid == 0 && mx >= 0x7F80u && a.status) atomicOr(a.status, SP24_STATUS_NONFINITE);
  } else {
    // ------------------------------------------------ grid barrier on amax
    if (tid == 0) {
      atomicMax(&a.ws[0], mx);
      __threadfence();
      atomicAdd(&a.ws[1], 1u);
      const uint64_t t0 = global_timer_ns();
      uint32_t polls = 0;
      while (ld_acquire_u32(&a.ws[1]) < gridDim.x) {
        __nanosleep(64);
        if ((++polls & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
          if (a.status) atomicOr(a.status, SP24_STATUS_TIMEOUT);
          break;
        }
      }
      const uint32_t amax = ld_acquire_u32(&a.ws[0]);
      s_amax = amax;
      __threadfence();
      if (atomicAdd(&a.ws[2], 1u) == gridDim.x - 1) {  // last to leave: reset the counters
        a.ws[0] = 0u;
        a.ws[1] = 0u;
        a.ws[2] = 0u;
        __threadfence();
      }
      if (blockIdx.x == 0) {
        if (amax >= 0x7F80u && a.status) atomicOr(a.status, SP24_STATUS_NONFINITE);
        if (a.scale_out) *a.scale_out = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
      }
    }
    named_bar_sync(1, kConsumers);
    const uint32_t amax = s_amax;
    const float s = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
    const bool direct = static_cast<int64_t>(n_my) * kChunkBytes < 2 * kTab * 2 * 8;
    if (!direct) build_table(tab, amax, s, tid);
    named_bar_sync(1, kConsumers);
    const CodeTable code{tab, (static_cast<int>(amax >> 7) - 23) * 128, s, direct};

    // ---------------------------------------------------------- phase 2
    for (int i = 0; i < n_my; ++i) {
      int slot = i;
      const int L = n_my + i;
      if (!resident) {
        slot = L % kStages;
        mbar_wait(&full[slot], static_cast<uint32_t>(L / kStages) & 1u, a.status);
      }
      const int64_t c = c0 + i;
      const int64_t nb = min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes);
      uint32_t mrow[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int off = (r * kConsumers + tid) * kUnit;
        const int64_t e0 = (c * kChunkBytes + off) / 2;
        mrow[r] = 0;
        if (off < nb) {
          if constexpr (OP == kOpPrune24) {
            mrow[r] = __ldcg(a.meta + e0 / 8);
          } else if constexpr (OP == kOpSlide68) {
            const uint8_t *mp = a.meta + 3 * (e0 / 16);
            mrow[r] = __ldcg(mp) | (static_cast<uint32_t>(__ldcg(mp + 1)) << 8) |
                      (static_cast<uint32_t>(__ldcg(mp + 2)) << 16);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int off = (r * kConsumers + tid) * kUnit;
        if (off < nb)
          phase2_unit<OP, DENSE>(ring + slot * kChunkBytes + off, (c * kChunkBytes + off) / 2, mrow[r], a,
                                 code);
      }
      __syncwarp();
      if (!resident && (tid & 31) == 0) mbar_arrive(&empty[slot]);
    }
  }
}

template <int OP, bool FP8, bool DENSE>
cudaError_t launch_stream_typed(const StreamArgs &a, int sm_count, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(stream_kernel<OP, FP8, DENSE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  const int64_t grid = a.nchunks < sm_count ? a.nchunks : sm_count;
  cfg.gridDim = dim3(static_cast<unsigned>(grid < 1 ? 1 : grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = FP8 ? 1 : 0;  // only the two-phase kernels wait on each other
  return cudaLaunchKernelEx(&cfg, stream_kernel<OP, FP8, DENSE>, a);
}

StreamArgs make_args(const void *x, int64_t nelem, uint32_t *ws, float *scale, int32_t *status,
                     void *out, uint8_t *meta, void *dense) {
  StreamArgs a;
  a.x = static_cast<const uint8_t *>(x);
  a.nbytes = nelem * 2;
  a.nchunks = (a.nbytes + kChunkBytes - 1) / kChunkBytes;
  a.ws = ws;
  a.scale_out = scale;
  a.status = status;
  a.out = static_cast<uint8_t *>(out);
  a.meta = meta;
  a.dense = static_cast<uint8_t *>(dense);
  return a;
}

}  // namespace

cudaError_t launch_quantize_fused(const void *x, int64_t nelem, uint32_t *ws, float *scale,
                                  uint8_t *q, int32_t *status, int sm_count, cudaStream_t st) {
  return launch_stream_typed<kOpQuantize, true, false>(
      make_args(x, nelem, ws, scale, status, q, nullptr, nullptr), sm_count, st);
}

cudaError_t launch_lift_fused(const void *x, int64_t nelem, uint32_t *ws, float *scale,
                              uint8_t *q, int32_t *status, int sm_count, cudaStream_t st) {
  return launch_stream_typed<kOpLift, true, false>(
      make_args(x, nelem, ws, scale, status, q, nullptr, nullptr), sm_count, st);
}

cudaError_t launch_prune24_fused(const void *w, int64_t nelem, bool fp8, uint32_t *ws,
                                 float *scale, void *values, uint8_t *meta, void *dense,
                                 int32_t *status, int sm_count, cudaStream_t st) {
  const StreamArgs a = make_args(w, nelem, ws, scale, status, values, meta, dense);
  if (fp8)
    return dense ? launch_stream_typed<kOpPrune24, true, true>(a, sm_count, st)
                 : launch_stream_typed<kOpPrune24, true, false>(a, sm_count, st);
  return dense ? launch_stream_typed<kOpPrune24, false, true>(a, sm_count, st)
               : launch_stream_typed<kOpPrune24, false, false>(a, sm_count, st);
}

cudaError_t launch_slide68_fused(const void *w, int64_t nelem, bool fp8, uint32_t *ws,
                                 float *scale, void *values, uint8_t *meta, int32_t *status,
                                 int sm_count, cudaStream_t st) {
  const StreamArgs a = make_args(w, nelem, ws, scale, status, values, meta, nullptr);
  return fp8 ? launch_stream_typed<kOpSlide68, true, false>(a, sm_count, st)
             : launch_stream_typed<kOpSlide68, false, false>(a, sm_count, st);
}

}  // namespace sp24
