// gemm.cu -- Y[M,N] = scale * X[M,K] . W[N,K]^T on the sm_100a tensor cores.
//
// W is the A operand of the MMA (128 rows per CTA, 2:4-compressed for the
// sparse kinds), the activations X are the B operand (BN tokens per CTA), so
// the fp32 accumulator tile lives in tensor memory as 128 lanes (W rows) x BN
// columns (tokens).  One CTA = 6 warps:
//   warp 0      TMA producer: W values, X tile and 2:4 metadata for each
//               K-stage into a ring of shared-memory stages (mbarrier
//               full/empty pairs);
//   warp 1      allocates tensor memory; one lane copies the stage's metadata
//               into TMEM (tcgen05.cp) and issues the tcgen05.mma(.sp)
//               instructions, releasing each stage with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld the accumulator, apply x_scale * w_scale,
//               round to bf16 and store Y (or, under split-K, store an fp32
//               partial and let the last CTA of the tile reduce in split order).
//
// 2:4 metadata in TMEM: for kind::f8f6f4 with M = 128 every accumulator lane
// (one W row) holds the 4-bit group descriptors of that row in K order, 64
// bits per K = 64 MMA step, i.e. exactly the row-major metadata bytes of the
// compressed layout.  Each stage's 128 rows x 16 bytes of metadata are one
// 128x128b tcgen05.cp into 4 TMEM columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace sp24 {

// ------------------------------------------------------------------ traits

template <int KIND>
struct KindTraits;

// 2:4 sparse E4M3: per stage 128 logical K = 64 value bytes + 16 metadata
// bytes per W row, 128 bytes per token; 2 MMAs of K = 64.
template <>
struct KindTraits<kSparseE4M3> {
  static constexpr bool kSparse = true;
  static constexpr int kBK = 128;
  static constexpr int kARowBytes = 64;
  static constexpr uint32_t kASwizzle = kSwizzle64B;
  static constexpr int kASbo = 8 * 64;
  static constexpr int kBRowBytes = 128;
  static constexpr int kERowBytes = 16;
  static constexpr int kMmas = 2;
  static constexpr int kAStep = 32;  // A bytes per MMA along K
  static constexpr int kBStep = 64;  // B bytes per MMA along K
  static constexpr uint32_t kFmt = 0;
  static constexpr int kAElemBytes = 1;
  static constexpr int kBElemBytes = 1;
  static constexpr int kBBoxElems = 128;     // one 128-byte swizzle row of X per box
  static constexpr bool kMetaTransform = false;
  static constexpr int kMetaColsPerMma = 2;  // 64 metadata bits per row per MMA
};

// Dense E4M3 (comparison kernel): 128 logical K per stage, 4 MMAs of K = 32.
template <>
struct KindTraits<kDenseE4M3> {
  static constexpr bool kSparse = false;
  static constexpr int kBK = 128;
  static constexpr int kARowBytes = 128;
  static constexpr uint32_t kASwizzle = kSwizzle128B;
  static constexpr int kASbo = 8 * 128;
  static constexpr int kBRowBytes = 128;
  static constexpr int kERowBytes = 0;
  static constexpr int kMmas = 4;
  static constexpr int kAStep = 32;
  static constexpr int kBStep = 32;
  static constexpr uint32_t kFmt = 0;
  static constexpr int kAElemBytes = 1;
  static constexpr int kBElemBytes = 1;
  static constexpr int kBBoxElems = 128;
  static constexpr bool kMetaTransform = false;
  static constexpr int kMetaColsPerMma = 0;
};

// 2:4 sparse BF16 (kind::f16): per stage 128 logical K = 64 bf16 values (128 B)
// + 16 metadata bytes per W row, 256 bytes (two 128-byte boxes) per token;
// 4 MMAs of K = 32.  For 16-bit operands the MMA reads the metadata of rows
// m and m + 8 from one TMEM lane (16 bits each), so the epilogue warps
// re-arrange each stage's metadata in shared memory before it is copied.
template <>
struct KindTraits<kSparseBF16> {
  static constexpr bool kSparse = true;
  static constexpr int kBK = 128;
  static constexpr int kARowBytes = 128;
  static constexpr uint32_t kASwizzle = kSwizzle128B;
  static constexpr int kASbo = 8 * 128;
  static constexpr int kBRowBytes = 256;
  static constexpr int kERowBytes = 16;
  static constexpr int kMmas = 4;
  static constexpr int kAStep = 32;  // 16 compressed bf16 per MMA
  static constexpr int kBStep = 64;  // 32 bf16 per MMA
  static constexpr uint32_t kFmt = 1;
  static constexpr int kAElemBytes = 2;
  static constexpr int kBElemBytes = 2;
  static constexpr int kBBoxElems = 64;
  static constexpr bool kMetaTransform = true;
  static constexpr int kMetaColsPerMma = 1;
};

template <int KIND, int BN>
struct Config {
  using T = KindTraits<KIND>;
  static constexpr uint32_t kABytes = 128 * T::kARowBytes;
  static constexpr uint32_t kBBytes = BN * T::kBRowBytes;
  static constexpr uint32_t kEBytes = 128 * T::kERowBytes;
  static constexpr uint32_t kTBytes = T::kMetaTransform ? 128 * 16 : 0;  // TMEM-ready metadata
  static constexpr uint32_t kTmaBytes = kABytes + kBBytes + kEBytes;
  static constexpr uint32_t kStageBytes = kTmaBytes + kTBytes;
  static constexpr int kBSub = T::kBRowBytes / 128;   // 128-byte X boxes per stage
  // Small token tiles run two CTAs per SM (more loads in flight for the
  // bandwidth-bound decode shapes); large ones one CTA with a deep ring.
  static constexpr int kCtasPerSm = BN <= 64 ? 2 : 1;
  static constexpr uint32_t kSmemBudget = kCtasPerSm == 2 ? 110 * 1024 : 220 * 1024;
  static constexpr int kStagesRaw = static_cast<int>(kSmemBudget / kStageBytes);
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 512 /*bars*/;
  static constexpr uint32_t kTmemNeed = BN + (T::kSparse ? 4 : 0);
  static constexpr uint32_t kTmemCols =
      kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
  static_assert(kStages >= 2, "shared-memory ring too shallow");
  static_assert(kStages * kStageBytes >= BN * 128 * 4, "split-K tile must fit in the idle ring");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be a multiple of 16 in [16,256]");
};

constexpr int kMaxSplits = 8;  // portable thread-block cluster size

struct GemmArgs {
  int M, N, K;
  int num_kb;
  int kb_per_split;
  int splits;
  uint16_t *y;
  const float *x_scale;
  const float *w_scale;
  int32_t *status;
};

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// ------------------------------------------------------------------ kernel

template <int KIND, int BN>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmE, const GemmArgs p) {
  using T = KindTraits<KIND>;
  using C = Config<KIND, BN>;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * C::kStageBytes);
  uint64_t *empty = full + S;
  uint64_t *meta_ready = empty + S;
  uint64_t *accum_bar = meta_ready + S;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int n0 = n_tile * 128;
  const int m0 = m_tile * BN;
  const int kb_begin = split * p.kb_per_split;
  const int kb_end = min(p.num_kb, kb_begin + p.kb_per_split);
  const int nkb = kb_end - kb_begin;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (T::kSparse) prefetch_tensormap(&tmE);
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&meta_ready[s], 128);
    }
    mbar_init(accum_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t keep_x = l2_policy_evict_last();    // X tiles are re-read by many CTAs
      const uint64_t stream_w = l2_policy_evict_first();  // weights are read once
      for (int i = 0; i < nkb; ++i) {
        const int s = i % S;
        const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
        if (i >= S && !mbar_wait(&empty[s], ph ^ 1u, p.status)) break;
        uint8_t *st = smem + s * C::kStageBytes;
        const int kb = kb_begin + i;
        mbar_arrive_expect_tx(&full[s], C::kTmaBytes);
        tma_load_2d(st, &tmA, &full[s], kb * (T::kARowBytes / T::kAElemBytes), n0, stream_w);
#pragma unroll
        for (int sub = 0; sub < C::kBSub; ++sub)
          tma_load_2d(st + C::kABytes + sub * BN * 128, &tmB, &full[s],
                      kb * (T::kBRowBytes / T::kBElemBytes) + sub * T::kBBoxElems, m0, keep_x);
        if (T::kSparse)
          tma_load_2d(st + C::kABytes + C::kBBytes, &tmE, &full[s], kb * T::kERowBytes, n0,
                      stream_w);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = mma_idesc(128, BN, T::kFmt, T::kSparse);
      const uint32_t d_tmem = tmem_base;
      const uint32_t e_tmem = tmem_base + BN;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % S;
        const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
        if (!mbar_wait(&full[s], ph, p.status)) break;
        if (T::kMetaTransform && !mbar_wait(&meta_ready[s], ph, p.status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_addr(smem + s * C::kStageBytes);
        const uint32_t b_addr = a_addr + C::kABytes;
        if (T::kSparse) {
          // 128 rows x 16 B, rows contiguous: core matrices of 8 rows are 128 B apart.
          const uint32_t e_addr = b_addr + C::kBBytes + (T::kMetaTransform ? C::kEBytes : 0);
          tmem_copy_128x128b(e_tmem, smem_desc(e_addr, 2048, 128, kSwizzleNone));
        }
#pragma unroll
        for (int kk = 0; kk < T::kMmas; ++kk) {
          const uint64_t ad = smem_desc(a_addr + kk * T::kAStep, 16, T::kASbo, T::kASwizzle);
          const uint32_t boff = (kk * T::kBStep / 128) * (BN * 128) + (kk * T::kBStep) % 128;
          const uint64_t bd = smem_desc(b_addr + boff, 16, 8 * 128, kSwizzle128B);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          if constexpr (KIND == kSparseE4M3) {
            mma_f8_sparse(d_tmem, ad, bd, idesc, e_tmem + 2 * kk, acc);
          } else if constexpr (KIND == kSparseBF16) {
            // one metadata column per MMA; columns are addressed in pairs and
            // the instruction descriptor's selector picks the column of the pair
            mma_bf16_sparse(d_tmem, ad, bd, idesc | static_cast<uint32_t>(kk & 1),
                            e_tmem + (kk & ~1), acc);
          } else {
            mma_f8_dense(d_tmem, ad, bd, idesc, acc);
          }
        }
        mma_commit(&empty[s]);
      }
      mma_commit(accum_bar);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;     // W row within the tile == accumulator lane
    const int n = n0 + row;
    if constexpr (T::kMetaTransform) {
      // Lane L = r0 + 8h + 16g of the TMEM metadata holds, for each of the
      // stage's 4 MMAs j, the 16 bits of K-half h of row 16g + r0 (low half)
      // and of row 16g + 8 + r0 (high half).
      const int t = threadIdx.x - 64;
      const int r0 = t & 7, h = (t >> 3) & 1, g = t >> 4;
      const int ra = 16 * g + r0, rb = ra + 8;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % S;
        const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
        if (!mbar_wait(&full[s], ph, p.status)) break;
        const uint8_t *e = smem + s * C::kStageBytes + C::kABytes + C::kBBytes;
        const uint16_t *ea = reinterpret_cast<const uint16_t *>(e + ra * 16);
        const uint16_t *eb = reinterpret_cast<const uint16_t *>(e + rb * 16);
        uint4 w;
        w.x = ea[0 + h] | (static_cast<uint32_t>(eb[0 + h]) << 16);
        w.y = ea[2 + h] | (static_cast<uint32_t>(eb[2 + h]) << 16);
        w.z = ea[4 + h] | (static_cast<uint32_t>(eb[4 + h]) << 16);
        w.w = ea[6 + h] | (static_cast<uint32_t>(eb[6 + h]) << 16);
        *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(e) + C::kEBytes + t * 16) = w;
        fence_proxy_async_smem();
        mbar_arrive(&meta_ready[s]);
      }
    }
    mbar_wait(accum_bar, 0, p.status);
    tc_fence_after();
    const float sx = p.x_scale ? __ldg(p.x_scale) : 1.0f;
    const float sw = p.w_scale ? __ldg(p.w_scale) : 1.0f;
    const float sc = sx * sw;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    if (p.splits == 1) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(t_row + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c + j;
          if (m < p.M) p.y[static_cast<size_t>(m) * p.N + n] = f32_to_bf16_bits(__uint_as_float(r[j]) * sc);
        }
      }
    } else {
      // Split-K: park this split's fp32 tile (valid token columns only) in
      // this CTA's shared memory, red[c * 128 + row]; the ring is idle now.
      float *red = reinterpret_cast<float *>(smem);
      const int mvalid = min(BN, p.M - m0);
#pragma unroll 1
      for (int c = 0; c < mvalid; c += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(t_row + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) red[(c + j) * 128 + row] = __uint_as_float(r[j]);
      }
    }
  }

  if (p.splits > 1) {
    // The K-splits of one output tile form a thread-block cluster.  After the
    // first cluster barrier every split's partial tile is in its CTA's shared
    // memory; CTA `rank` then reduces the token columns c = rank (mod splits),
    // reading all partials through distributed shared memory in split order
    // (deterministic), and the second barrier keeps every CTA's shared memory
    // alive until its peers have finished reading it.
    cluster_sync_all();
    if (warp >= 2) {
      const int q = warp & 3;
      const int row = q * 32 + lane;
      const int n = n0 + row;
      const int S2 = p.splits;
      const uint32_t rank = cluster_ctarank();
      const int mvalid = min(BN, p.M - m0);
      const float sx = p.x_scale ? __ldg(p.x_scale) : 1.0f;
      const float sw = p.w_scale ? __ldg(p.w_scale) : 1.0f;
      const float sc = sx * sw;
      const uint32_t red_base = smem_addr(smem) + static_cast<uint32_t>(row) * 4u;
#pragma unroll 1
      for (int c = static_cast<int>(rank); c < mvalid; c += S2) {
        const uint32_t local = red_base + static_cast<uint32_t>(c) * 128u * 4u;
        float v[kMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2)
          v[s2] = s2 < S2 ? ld_dsmem_f32(dsmem_map(local, static_cast<uint32_t>(s2))) : 0.0f;
        float acc = 0.0f;
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2) acc += v[s2];
        p.y[static_cast<size_t>(m0 + c) * p.N + n] = f32_to_bf16_bits(acc * sc);
      }
    }
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major 2-D map: `inner` elements per row (contiguous), `outer` rows.
static bool make_map(CUtensorMap *map, const void *ptr, CUtensorMapDataType dt, int elem_bytes,
                     uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int choose_bn(GemmKind kind, int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128 || kind == kSparseBF16) return 128;  // bf16 X stages are twice as large
  return 256;
}

static int ctas_per_sm(int bn) { return bn <= 64 ? 2 : 1; }

GemmPlan plan_gemm(GemmKind kind, int M, int N, int K, int sm_count) {
  GemmPlan pl{};
  pl.bn = choose_bn(kind, M);
  pl.bk = 128;
  pl.tiles_n = N / 128;
  pl.tiles_m = (M + pl.bn - 1) / pl.bn;
  pl.num_kb = K / pl.bk;
  const int tiles = pl.tiles_n * pl.tiles_m;
  const int slots = sm_count * ctas_per_sm(pl.bn);
  pl.kb_per_split = pl.num_kb;
  pl.splits = 1;
  if (tiles * 2 <= slots) {
    // Split K over a cluster of up to 8 CTAs so that the CTAs fill the
    // machine; each split keeps >= 4 pipeline stages of work.
    double best = -1.0;
    for (int kps = pl.num_kb; kps >= 4; --kps) {
      const int s = (pl.num_kb + kps - 1) / kps;
      if (s > kMaxSplits) break;
      const long units = static_cast<long>(tiles) * s;
      const long waves = (units + slots - 1) / slots;
      const double eff = static_cast<double>(units) / static_cast<double>(waves * slots);
      if (eff > best + 1e-9) {
        best = eff;
        pl.kb_per_split = kps;
        pl.splits = s;
      }
    }
  }
  pl.partial_bytes = 0;
  pl.counter_bytes = 0;
  return pl;
}

template <int KIND, int BN>
static cudaError_t launch_typed(const GemmPlan &pl, const void *xq, const float *x_scale,
                                const void *w_values, const uint8_t *w_meta, const float *w_scale,
                                void *y, int M, int N, int K, void *workspace, int32_t *status,
                                cudaStream_t st) {
  using T = KindTraits<KIND>;
  using C = Config<KIND, BN>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(gemm_kernel<KIND, BN>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;

  CUtensorMap tmA, tmB, tmE;
  const CUtensorMapDataType dtA =
      T::kAElemBytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapDataType dtB =
      T::kBElemBytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint64_t a_row = T::kSparse ? static_cast<uint64_t>(K) / 2 : static_cast<uint64_t>(K);
  const CUtensorMapSwizzle a_sw =
      T::kASwizzle == kSwizzle64B ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_map(&tmA, w_values, dtA, T::kAElemBytes, a_row, N, T::kARowBytes / T::kAElemBytes,
                128, a_sw))
    return cudaErrorInvalidValue;
  if (!make_map(&tmB, xq, dtB, T::kBElemBytes, K, M, T::kBBoxElems, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (T::kSparse) {
    if (!make_map(&tmE, w_meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(K) / 8, N,
                  16, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    tmE = tmA;  // unused
  }
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.num_kb = pl.num_kb;
  a.kb_per_split = pl.kb_per_split;
  a.splits = pl.splits;
  a.y = static_cast<uint16_t *>(y);
  a.x_scale = x_scale;
  a.w_scale = w_scale;
  a.status = status;
  (void)workspace;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.tiles_n, pl.tiles_m, pl.splits);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(pl.splits);
  cfg.attrs = attr;
  cfg.numAttrs = pl.splits > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<KIND, BN>, tmA, tmB, tmE, a);
}

template <int KIND>
static cudaError_t launch_kind(const GemmPlan &pl, const void *xq, const float *x_scale,
                               const void *w_values, const uint8_t *w_meta, const float *w_scale,
                               void *y, int M, int N, int K, void *ws, int32_t *status,
                               cudaStream_t st) {
  switch (pl.bn) {
    case 16: return launch_typed<KIND, 16>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    case 32: return launch_typed<KIND, 32>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    case 64: return launch_typed<KIND, 64>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    case 128: return launch_typed<KIND, 128>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    case 256: return launch_typed<KIND, 256>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(GemmKind kind, const GemmPlan &pl, const void *xq, const float *x_scale,
                        const void *w_values, const uint8_t *w_meta, const float *w_scale,
                        void *y, int M, int N, int K, void *workspace, int32_t *status,
                        cudaStream_t st) {
  switch (kind) {
    case kSparseE4M3:
      return launch_kind<kSparseE4M3>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    case kDenseE4M3:
      return launch_kind<kDenseE4M3>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    case kSparseBF16:
      return launch_kind<kSparseBF16>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace sp24
