// gemm.cu -- Y[M,N] = scale * X[M,K] . W[N,K]^T on the sm_100a tensor cores.
//
// W is the A operand of the MMA (128 rows per CTA, 2:4-compressed for the
// sparse kinds), the activations X are the B operand (BN tokens per CTA), so
// the fp32 accumulator tile lives in tensor memory as 128 lanes (W rows) x BN
// columns (tokens).  One CTA = 6 warps (10 for two-row-tile tiles):
//   warp 0      TMA producer: W values, X tile and 2:4 metadata for each
//               K-stage into a ring of shared-memory stages (mbarrier
//               full/empty pairs);
//   warp 1      allocates tensor memory; one lane copies the stage's metadata
//               into TMEM (tcgen05.cp) and issues the tcgen05.mma(.sp)
//               instructions, releasing each stage with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld the accumulator, apply x_scale * w_scale,
//   (2-9)       round to bf16 and store Y (stream-K: see GemmArgs).
// The kernel is persistent: one CTA per SM walks a list of (tile, k-range)
// segments; two TMEM accumulators (when they fit) let the epilogue of one
// segment overlap the main loop of the next.
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
#include "quant_common.cuh"
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
  static constexpr uint32_t kDFmt = 1;       // fp32 accumulator
  static constexpr int kAElemBytes = 1;
  static constexpr int kBElemBytes = 1;
  static constexpr int kBBoxElems = 128;     // one 128-byte swizzle row of X per box
  static constexpr bool kMetaTransform = false;
  static constexpr int kMetaColsPerMma = 2;  // 64 metadata bits per row per MMA
  static constexpr bool kPacked = false;
  static constexpr bool kFp4 = false;
  static constexpr bool kPair = false;
};

// The same MMA with the weights in the tile-packed layout: each stage's
// values (already in the 64-byte-swizzled shared-memory order) and metadata
// are one contiguous 10240-byte block, fetched with a single bulk copy.
template <>
struct KindTraits<kSparseE4M3Packed> : KindTraits<kSparseE4M3> {
  static constexpr bool kPacked = true;
};

// INT8 W8A8 (kind::i8): the packed layout and the 8-bit 2:4 metadata of the
// E4M3 kind, signed operands, an s32 accumulator converted to fp32 in the
// epilogue.
template <>
struct KindTraits<kSparseI8Packed> : KindTraits<kSparseE4M3Packed> {
  static constexpr uint32_t kFmt = 1;   // signed 8-bit
  static constexpr uint32_t kDFmt = 2;  // s32 accumulator
};

// The packed E4M3 kind on SM pairs (tensor-bound tiles): a cluster of two
// CTAs runs one M = 256 sparse MMA per K step (cta_group::2).  Each CTA
// loads the packed blocks of its own 128 weight rows (through a 2-D tensor
// map over the packed buffer: a 10240-byte block is 40 rows of 256 bytes)
// and half of the activation tile, both counted on the even CTA's barrier;
// the even CTA issues the metadata copies, MMAs and commits for both, and
// each CTA drains the accumulator of its own rows.  Against one CTA holding
// two row tiles the shared-memory bytes per MMA are the same, but each
// CTA's accumulator is BN columns, so two fit tensor memory and a tile's
// epilogue overlaps the next tile's main loop.
template <>
struct KindTraits<kSparseE4M3Pair> : KindTraits<kSparseE4M3Packed> {
  static constexpr bool kPair = true;
};

// 2:4 sparse FP4 (E2M1 A and B, kind::f8f6f4): the codes are packed two per
// byte in global memory and loaded with 4-bit tensor maps
// (CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B), which lay every 16 codes out in 16
// bytes of shared memory (8 bytes of codes, 8 of padding): the byte geometry
// of the E4M3 tiles, one byte per element.  Such a box is 128 elements wide,
// so a stage covers two 128-K blocks (KB = 2): 128 stored values = 128
// bytes per W row (128-byte swizzle), 2 x 128 bytes per token, and the two
// blocks' metadata (16 bytes per row each, two 2 KB boxes).
template <>
struct KindTraits<kSparseFP4> : KindTraits<kSparseE4M3> {
  static constexpr uint32_t kASwizzle = kSwizzle128B;
  static constexpr int kASbo = 8 * 128;  // 8 rows of one stage's 128 bytes
  static constexpr uint32_t kFmt = 5;     // E2M1
  static constexpr bool kFp4 = true;
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
  static constexpr uint32_t kDFmt = 1;
  static constexpr int kAElemBytes = 1;
  static constexpr int kBElemBytes = 1;
  static constexpr int kBBoxElems = 128;
  static constexpr bool kMetaTransform = false;
  static constexpr int kMetaColsPerMma = 0;
  static constexpr bool kPacked = false;
  static constexpr bool kFp4 = false;
  static constexpr bool kPair = false;
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
  static constexpr uint32_t kDFmt = 1;
  static constexpr int kAElemBytes = 2;
  static constexpr int kBElemBytes = 2;
  static constexpr int kBBoxElems = 64;
  static constexpr bool kMetaTransform = true;
  static constexpr int kMetaColsPerMma = 1;
  static constexpr bool kPacked = false;
  static constexpr bool kFp4 = false;
  static constexpr bool kPair = false;
};

// MT = 128-row W tiles per CTA tile (1 or 2).  With MT = 2 each stage
// carries two weight tiles and one activation tile, and every k-block issues
// the MMAs of both row tiles against the same activation tile: the same
// activation bytes feed twice the tensor work, which is what bounds large
// token tiles (operand ingest into shared memory, not the tensor pipe).
//
// KB = 128-K blocks per pipeline stage (1 or 2).  Decode-sized tiles do
// little tensor work per stage, so the fixed cost of a stage (barrier wait,
// metadata copy, commit, each issued by one thread) bounds their main loop;
// two blocks per stage halve it.  Packed weights only: the stage's two
// blocks of a row tile are adjacent in memory (one bulk copy) and their
// metadata is one 128x256b copy.
// Staged activation codes of the fused local quantisation (BN = 16 kernels):
// up to this many bytes of E4M3 codes kept in shared memory.
constexpr uint32_t kXStageBytes = 8192;

template <int KIND, int BN, int MT = 1, int KB = 1, int XQ = 0>
struct Config {
  using T = KindTraits<KIND>;
  static_assert(KB == 1 || (KB == 2 && (T::kPacked || T::kFp4) && MT == 1),
                "two-block stages are for packed or FP4, one-row-tile tiles");
  static_assert(!T::kFp4 || (KB == 2 && MT == 1), "FP4 stages are two 128-K blocks of one row tile");
  static constexpr int kRows = 128 * MT;
  static constexpr uint32_t kABytes = kRows * T::kARowBytes * KB;
  static_assert(!T::kPair || (MT == 1 && XQ == 0 && BN >= 128 && BN % 32 == 0),
                "SM pairs run one-row-tile stages of wide token tiles");
  static constexpr int kBRows = T::kPair ? BN / 2 : BN;  // activation rows this CTA loads
  static constexpr uint32_t kBBytes = kBRows * T::kBRowBytes * KB;
  static constexpr uint32_t kEBytes = kRows * T::kERowBytes * KB;
  static constexpr uint32_t kTBytes = T::kMetaTransform ? 128 * 16 : 0;  // TMEM-ready metadata
  // Transaction bytes of a stage's copies: a 4-bit box moves its packed
  // bytes (half its shared-memory footprint, which pads every 8 bytes of
  // codes to 16).
  static constexpr uint32_t kTmaBytes = (T::kFp4 ? (kABytes + kBBytes) / 2 : kABytes + kBBytes) + kEBytes;
  static constexpr uint32_t kWBytes = kABytes + kEBytes;  // the weight half of a stage
  // shared-memory footprint of a stage (the padded size for 4-bit boxes)
  static constexpr uint32_t kStageBytes = kABytes + kBBytes + kEBytes + kTBytes;
  static constexpr int kBSub = T::kBRowBytes * KB / 128;  // 128-byte X boxes per stage
  static constexpr int kMmas = T::kMmas * KB;             // MMAs per row tile per stage
  // Stage layout: [A][B][E][T] (tensor-mapped weights; A and E hold all kRows
  // rows, row tile i at 128 i rows) or [A0 E0 (A0' E0')][A1 E1][B] (packed:
  // each row tile's values and metadata arrive together in one bulk copy,
  // the KB blocks of a row tile back to back).
  static constexpr uint32_t kBOff = T::kPacked ? MT * KB * kPackedBlockBytes : kABytes;
  static constexpr uint32_t kEOff = T::kPacked ? 128 * T::kARowBytes : kABytes + kBBytes;
  __host__ __device__ static constexpr uint32_t a_off(int i) {
    return T::kPacked ? i * KB * kPackedBlockBytes : i * 128 * T::kARowBytes;
  }
  __host__ __device__ static constexpr uint32_t e_off(int i) {
    return T::kPacked ? i * KB * kPackedBlockBytes + 128 * T::kARowBytes : kEOff + i * 128 * T::kERowBytes;
  }
  // Persistent CTAs.  Small token tiles (decode shapes, stream-K) keep the
  // footprint to half an SM, so that the next kernel's CTAs can already be
  // resident, and streaming weights, while this kernel drains; large tiles
  // take the whole SM for a deep ring.
  // Epilogue warps: two per TMEM lane quarter for two-row-tile tiles (one
  // per row tile), whose single accumulator leaves the epilogue exposed
  // between main loops; one per quarter otherwise.
  static constexpr int kEpiWarps = MT == 2 ? 8 : 4;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kThreads = 64 + kEpiThreads;
  static constexpr int kRtPerWarp = MT * 4 / kEpiWarps;  // row tiles each epilogue warp drains
  static constexpr uint32_t kSmemBudget = BN <= 64 ? 108 * 1024 : (kEpiWarps == 8 ? 224 * 1024 : 214 * 1024);
  // Decode-sized tiles: two CTAs must fit an SM (shared memory above, and
  // registers: at most 65536 / (2 * kThreads) per thread), or the next
  // kernel cannot start streaming its weights before this one ends.
  static constexpr int kMinBlocks = BN <= 64 ? 2 : 1;
  // Wide token tiles write Y through shared memory: each epilogue warp
  // stages its 32 rows x 32 tokens of a pass (2 KB of bf16) in one of two
  // buffers of its own and stores them with a 2-D bulk tensor copy, so the
  // warps never wait for each other (scattered 2-byte stores into Y rows cost
  // ~10 us per 128 x 224 tile).  Decode-sized tiles (BN <= 64) keep direct
  // stores and the deeper ring.
  static constexpr bool kTmaStoreY = BN >= 128;
  static constexpr uint32_t kStageY = 32 * 32 * 2;          // one warp's pass
  static constexpr uint32_t kYBytes = kTmaStoreY ? kEpiWarps * 2 * kStageY : 0;
  static constexpr uint32_t kXStage = (XQ != 0 && BN == 16) ? kXStageBytes : 0;
  static constexpr int kStagesRaw = static_cast<int>((kSmemBudget - kYBytes - kXStage) / kStageBytes);
  static constexpr int kStages = kStagesRaw > 16 ? 16 : kStagesRaw;
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + kYBytes + kXStage + 1024 /*align*/ + 1024 /*bars*/;
  // Accumulators: MT x BN columns each; two of them (the epilogue of one
  // output tile overlaps the main loop of the next) whenever they fit in the
  // 512 TMEM columns next to the 4 metadata columns per row tile.
  static constexpr uint32_t kMetaCols = T::kSparse ? 4 * MT * KB : 0;
  static constexpr int kAccBufs = (2 * MT * BN + kMetaCols <= 512) ? 2 : 1;
  static constexpr uint32_t kAccCols = MT * BN;
  static constexpr uint32_t kTmemNeed = kAccBufs * kAccCols + kMetaCols;
  static constexpr uint32_t kTmemCols =
      kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
  static_assert(kStages >= 2, "shared-memory ring too shallow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be a multiple of 16 in [16,256]");
  static_assert(MT == 1 || MT == 2, "one or two 128-row W tiles per CTA tile");
  static_assert(MT == 1 || !T::kMetaTransform, "the BF16 metadata re-layout handles one row tile");
  static_assert(kTmemNeed <= 512, "accumulators and metadata exceed tensor memory");
  static_assert(kBOff % 1024 == 0 && kStageBytes % 1024 == 0, "128-byte-swizzled tiles need 1 KB alignment");
  static constexpr int kEpiCols = BN % 32 == 0 ? 32 : 16;  // token columns per epilogue pass
  static_assert(!kTmaStoreY || kEpiCols == 32, "staged Y passes are 32 tokens wide");
};

// Work decomposition ("data-parallel + stream-K").  The first dp_tiles tiles
// are taken whole: CTA g gets tiles g, g + G, ...  The remaining sk_tiles
// tiles are cut into (tile, k-block) units u = t * num_kb + kb, and CTA
// g < sk_grid takes the contiguous range [g U / sk_grid, (g + 1) U / sk_grid),
// so the leftover work is spread evenly instead of forming a partial wave.
// A tile split between CTAs is finished by the CTA that computed its k-block
// 0 (the owner): the others (contributors) leave fp32 partial tiles in the
// workspace and count themselves in the tile's counter; the owner waits for
// them, adds the partials in CTA order (deterministic) and writes Y.  A CTA's
// only contributor segment is the first of its range, so it never waits for
// anybody and owners always make progress.
struct GemmArgs {
  int M, N, K;
  int num_kb;
  int tiles_n;
  int num_tiles;
  int dp_tiles;        // tiles taken whole
  int sk_grid;         // CTAs sharing the stream-K units
  int64_t sk_units;    // (num_tiles - dp_tiles) * num_kb
  uint16_t *y;
  const float *x_scale;
  const float *w_scale;
  float *partials;     // stream-K: [sk_grid][128 MT][BN] fp32
  uint32_t *counters;  // stream-K: [num_tiles - dp_tiles], zero between calls
  int32_t *status;
  const uint8_t *packed;  // tile-packed weights (packed kind only)
  // Fused activation quantisation (XQ != 0): bf16 X of xvec 8-element
  // vectors in, its E4M3 codes (lifted for XQ = 2) out to xq, which is the
  // B operand the kernel then loads.
  const uint16_t *x;
  uint8_t *xq;
  float *x_scale_out;
  int64_t xvec;
  int xstaged;  // codes staged in shared memory (kXStage)
  // Scale vectors (VS kernels): x_scale holds M per-token scales when x_vec,
  // w_scale N per-channel scales when w_vec; otherwise one value each.
  int x_vec, w_vec;
};

enum SegRole : int { kWhole = 0, kOwner = 1, kContrib = 2 };

struct Segment {
  int tile, kb0, kb1, role;
};

// `me` / `ncta`: this CTA's index and the count of schedule units (CTAs,
// or SM pairs for the pair kind).
struct SegIter {
  int64_t u, u_end;
  int tile, step;
  __device__ __forceinline__ void init(const GemmArgs &p, int me, int ncta) {
    tile = me;
    step = ncta;
    u = u_end = 0;
    if (me < p.sk_grid) {
      u = static_cast<int64_t>(me) * p.sk_units / p.sk_grid;
      u_end = static_cast<int64_t>(me + 1) * p.sk_units / p.sk_grid;
    }
  }
  __device__ __forceinline__ bool next(const GemmArgs &p, Segment &s) {
    if (tile < p.dp_tiles) {
      s.tile = tile;
      s.kb0 = 0;
      s.kb1 = p.num_kb;
      s.role = kWhole;
      tile += step;
      return true;
    }
    if (u >= u_end) return false;
    s.tile = p.dp_tiles + static_cast<int>(u / p.num_kb);
    s.kb0 = static_cast<int>(u % p.num_kb);
    s.kb1 = static_cast<int>(min(static_cast<int64_t>(p.num_kb), s.kb0 + (u_end - u)));
    s.role = s.kb0 != 0 ? kContrib : (s.kb1 == p.num_kb ? kWhole : kOwner);
    u += s.kb1 - s.kb0;
    return true;
  }
};

// CTA whose stream-K range holds unit u.
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t units, int grid) {
  return static_cast<int>(((u + 1) * grid + units - 1) / units) - 1;
}

// An accumulator word as fp32: the bits themselves, or (kind::i8) the s32
// sum converted (exact below 2^24, correctly rounded above).
template <int KIND>
__device__ __forceinline__ float acc_f32(uint32_t v) {
  if constexpr (KIND == kSparseI8Packed)
    return __int2float_rn(static_cast<int>(v));
  else
    return __uint_as_float(v);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ void red_release_add_gpu(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_max_relaxed_gpu(uint32_t *p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spin (bounded) until *p reaches `expect`; acquire semantics.
__device__ __forceinline__ void wait_count_gpu(const uint32_t *p, uint32_t expect, int32_t *status) {
  const uint64_t t0 = global_timer_ns();
  uint32_t polls = 0;
  while (ld_acquire_gpu(p) < expect) {
    __nanosleep(32);
    if ((++polls & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
      if (status) atomicOr(status, SP24_STATUS_TIMEOUT);
      break;
    }
  }
}

// Per-tensor E4M3 quantisation of the activations fused in front of the
// GEMM (X of at most kFusedXVec 8-element vectors: decode batches of a few
// tokens), run by the 128 epilogue threads (t = 0..127) while the producer
// already streams weights.  Every CTA takes the amax of all of X and encodes
// all of it itself (each thread holds up to kXReg 16-byte vectors in
// registers), so no CTA waits for another: s = amax / 448 (1 when amax = 0),
// codes E4M3(RN_fp32(x / s)) by e4m3_codes8_fast, which equals the correctly
// rounded division on every input (e4m3_codes8_div where it cannot decide).
// When the codes fit kXStageBytes (`xstage`, BN = 16 kernels) they go to
// shared memory, from where the producer copies each stage's rows into its B
// tile, and only CTA 0 writes them to xq for the caller; otherwise every CTA
// writes the (identical) codes to xq and its producer TMA-loads them.  Either
// way the producer waits for this CTA only (x_ready).
// XQ = 2 writes the SlideSparse lift: each 8-group g of a row becomes the 12
// codes of windows 2j..2j+3, j = 0..2.  Returns s.
constexpr int kXReg = 8;
static_assert(kFusedXVec <= 128 * kXReg, "every thread holds its vectors of X in registers");

template <int XQ>
__device__ __forceinline__ void store_xvec(uint8_t *dst, int64_t v, const uint2 c) {
  if constexpr (XQ == 1) {
    *reinterpret_cast<uint2 *>(dst + 8 * v) = c;
  } else {
    uint32_t *o = reinterpret_cast<uint32_t *>(dst + 12 * v);
    o[0] = c.x;
    o[1] = __byte_perm(c.x, c.y, 0x5432);  // codes 2..5
    o[2] = c.y;
  }
}

template <int XQ>
__device__ float fused_quantize(const GemmArgs &p, int t, uint32_t *s_red, float *s_scale, uint64_t *x_ready,
                                uint8_t *xstage) {
  const int64_t nvec = p.xvec;
  const uint4 *xv = reinterpret_cast<const uint4 *>(p.x);
  // vectors t + 128 u, u < kXReg: all loads in flight at once, kept
  uint4 w[kXReg];
#pragma unroll
  for (int u = 0; u < kXReg; ++u)
    w[u] = t + 128 * u < nvec ? __ldg(xv + t + 128 * u) : make_uint4(0u, 0u, 0u, 0u);
  uint32_t m2 = 0;
#pragma unroll
  for (int u = 0; u < kXReg; ++u) m2 = __vmaxu2(m2, absmax8x2(w[u]));
  const uint32_t mw = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
  if ((t & 31) == 0) s_red[t >> 5] = mw;
  named_bar_sync(1, 128);
  if (t == 0) {
    const uint32_t amax = max(max(s_red[0], s_red[1]), max(s_red[2], s_red[3]));
    const float sx = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
    if (blockIdx.x == 0) {
      if (amax >= 0x7F80u && p.status) atomicOr(p.status, SP24_STATUS_NONFINITE);
      *p.x_scale_out = sx;
    }
    s_scale[0] = sx;
    s_scale[1] = __frcp_rn(sx);
  }
  named_bar_sync(1, 128);
  const float sx = s_scale[0], rx = s_scale[1];
  uint8_t *dst = xstage ? xstage : p.xq;
  const bool also_out = xstage && blockIdx.x == 0;  // staged codes: CTA 0 returns them
  // this thread's nv vectors, encoded two at a time (the pairs interleave; no
  // work for absent vectors)
  const int64_t mine = nvec - t;
  const int nv = mine <= 0 ? 0 : static_cast<int>(mine >= 128 * kXReg ? kXReg : (mine + 127) / 128);
#pragma unroll
  for (int u = 0; u < kXReg; u += 2) {
    if (u < nv) {
      bool ok0, ok1;
      uint2 c0 = e4m3_codes8_fast(w[u], rx, ok0);
      uint2 c1 = e4m3_codes8_fast(w[u + 1], rx, ok1);
      if (!ok0) c0 = e4m3_codes8_div(w[u], sx);
      if (!ok1) c1 = e4m3_codes8_div(w[u + 1], sx);
      const int64_t v = t + 128 * u;
      store_xvec<XQ>(dst, v, c0);
      if (also_out) store_xvec<XQ>(p.xq, v, c0);
      if (u + 1 < nv) {
        store_xvec<XQ>(dst, v + 128, c1);
        if (also_out) store_xvec<XQ>(p.xq, v + 128, c1);
      }
    }
  }
  if (!xstage) fence_proxy_async_global();  // the codes are read back by TMA loads
  named_bar_sync(1, 128);
  if (t == 0) mbar_arrive(x_ready);
  return sx;
}

// Scale of token m for the VS epilogue: the per-token vector, or the single
// scale (0 for the padding tokens past M, which are never stored).
__device__ __forceinline__ float token_scale(const GemmArgs &p, int m, float sx) {
  if (!p.x_vec) return sx;
  return m < p.M ? __ldg(p.x_scale + m) : 0.0f;
}

// ------------------------------------------------------------------ kernel

template <int KIND, int BN, int MT, int XQ, int KB, bool VS>
__global__ void __launch_bounds__(Config<KIND, BN, MT, KB, XQ>::kThreads, Config<KIND, BN, MT, KB, XQ>::kMinBlocks)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                const GemmArgs p) {
  using T = KindTraits<KIND>;
  using C = Config<KIND, BN, MT, KB, XQ>;
  constexpr int S = C::kStages;
  constexpr int NB = C::kAccBufs;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ystage = smem + S * C::kStageBytes;  // kYBytes: two staged Y passes
  uint8_t *xstage = ystage + C::kYBytes;         // kXStage: staged activation codes
  uint64_t *full = reinterpret_cast<uint64_t *>(xstage + C::kXStage);
  uint64_t *empty = full + S;
  uint64_t *meta_ready = empty + S;
  uint64_t *tmem_full = meta_ready + S;
  uint64_t *tmem_empty = tmem_full + NB;
  uint64_t *x_ready = tmem_empty + NB;  // fused quantisation: codes written
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(x_ready + 1);
  [[maybe_unused]] __shared__ uint32_t s_xred[4];
  [[maybe_unused]] __shared__ float s_xscale[2];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (p.num_tiles + p.tiles_n - 1) / p.tiles_n;
  // SM pairs: rank in the pair (0 = the CTA that issues the MMAs) and the
  // pair's index in the schedule
  const uint32_t rank = T::kPair ? cluster_ctarank() & 1u : 0u;
  const int me = T::kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int ncta = T::kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // first weight row of a tile held by this CTA
  auto row0 = [&](int tile) {
    return T::kPair ? (tile % p.tiles_n) * 256 + static_cast<int>(rank) * 128 : (tile % p.tiles_n) * C::kRows;
  };

  if (warp == 0 && lane == 0) {
    if (!T::kPacked || T::kPair) prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (T::kSparse && !T::kPacked) prefetch_tensormap(&tmE);
    if (C::kTmaStoreY) prefetch_tensormap(&tmY);
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&meta_ready[s], 128);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], T::kPair ? 2 * C::kEpiThreads : C::kEpiThreads);  // pairs: both CTAs drain
    }
    mbar_init(x_ready, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (T::kPair) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // pairs: both CTAs' barriers exist before the first remote arrive or load
  if constexpr (T::kPair) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Programmatic dependent launch.  This grid may start while the previous
  // kernel in the stream is still running.  Compressed weights are only ever
  // written by the weight-path kernels (prune/compress, decompose), which do
  // not release their dependents early, so the producer may stream weight
  // tiles right away; activations, scales and Y are touched only after
  // griddepcontrol.wait, i.e. after the previous kernel has completed.
  if (warp != 0) grid_dependency_wait();
  grid_launch_dependents();

  // The producer and MMA warps walk the schedule with all 32 lanes, combine
  // their barrier waits by vote and issue every TMA / tcgen05 instruction
  // from one elected lane: the loop counters, addresses and descriptors are
  // then warp-uniform, which the issue of those instructions needs to be
  // cheap.
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    {
      const bool leader = elect_one();
      const uint64_t keep_x = l2_policy_evict_last();  // X tiles are re-read by many CTAs
      // Weights are read once when there is a single token tile; otherwise
      // every token tile re-reads them and they should stay in L2.
      const uint64_t stream_w = tiles_m == 1 ? l2_policy_evict_first() : l2_policy_evict_normal();
      // weight half of a stage: values + metadata of rows n0.., k-block kb
      auto load_weights = [&](uint8_t *st, uint64_t *bar, int n0, int kb) {
        if constexpr (T::kPair) {
          // this CTA's packed block (rows n0..n0+127, k-block kb): rows of
          // 256 bytes 40 (blk) .. 40 (blk) + 39 of the packed tensor map,
          // counted on the even CTA's barrier
          const int blk = ((n0 / 128) * p.num_kb + kb) * KB;
          tma_load_2d_pair(st, &tmA, mapa_shared(bar, 0u), 0, blk * (kPackedBlockBytes / 256), stream_w);
        } else if constexpr (T::kPacked) {
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            const uint8_t *blk = p.packed +
                                 ((static_cast<int64_t>(n0 / 128 + i) * p.num_kb + kb) * KB) * kPackedBlockBytes;
            bulk_load_g2s(st + C::a_off(i), blk, KB * kPackedBlockBytes, bar, stream_w);
          }
        } else if constexpr (T::kFp4) {
          // stage kb = stored codes 128 kb .. 128 kb + 127 of each row (one
          // 4-bit box), and the metadata of 128-K blocks 2 kb, 2 kb + 1
          tma_load_2d(st, &tmA, bar, kb * 128, n0, stream_w);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tma_load_2d(st + C::kEOff + j * 128 * T::kERowBytes, &tmE, bar, (2 * kb + j) * T::kERowBytes, n0,
                        stream_w);
        } else {
          tma_load_2d(st, &tmA, bar, kb * (T::kARowBytes / T::kAElemBytes), n0, stream_w);
          if (T::kSparse) tma_load_2d(st + C::kEOff, &tmE, bar, kb * T::kERowBytes, n0, stream_w);
        }
      };
      // Staged activation codes (fused local quantisation): the producer
      // copies each stage's X rows from shared memory into the stage's B tile
      // (the 128-byte swizzle: 16-byte chunk c of row m at c ^ (m & 7)); the
      // rows past M are left as they are, since they only feed output
      // columns that are never stored.
      const bool staged = C::kXStage > 0 && p.xstaged;
      auto copy_x_rows = [&](uint8_t *st, int kb) {
        for (int q = lane; q < p.M * KB * 8; q += 32) {
          const int c = q & 7, u = (q >> 3) % KB, m = q / (8 * KB);
          const uint4 v = *reinterpret_cast<const uint4 *>(xstage + static_cast<int64_t>(m) * p.K +
                                                           (kb * KB + u) * 128 + c * 16);
          *reinterpret_cast<uint4 *>(st + C::kBOff + u * BN * 128 + m * 128 + ((c ^ (m & 7)) * 16)) = v;
        }
        fence_proxy_async_smem();  // generic writes, read by the MMA (async proxy)
        __syncwarp();
      };
      // Pass 1 (before the grid dependency resolves): the weight half of the
      // first S stages (with staged codes the stage's arrival waits for the
      // X copy: only the transaction bytes are announced here).  Pass 2:
      // everything else, in the same stage order.
      SegIter it;
      it.init(p, me, ncta);
      Segment sg;
      int i = 0;
      bool ok = true;
      int pre = 0;  // stages whose weight tiles were issued ahead
      {
        SegIter it0;
        it0.init(p, me, ncta);
        Segment s0;
        while (pre < S && it0.next(p, s0)) {
          const int n0 = row0(s0.tile);
          for (int kb = s0.kb0; kb < s0.kb1 && pre < S; ++kb, ++pre) {
            uint8_t *st = smem + pre * C::kStageBytes;
            if (leader) {
              if (staged)
                mbar_expect_tx(&full[pre], C::kWBytes);
              else if (!T::kPair || rank == 0)  // pairs: the even CTA expects both CTAs' bytes
                mbar_arrive_expect_tx(&full[pre], T::kPair ? 2 * C::kTmaBytes : C::kTmaBytes);
              load_weights(st, &full[pre], n0, kb);
            }
          }
        }
      }
      // The rest of this CTA's weights, when they are read once (a single
      // token tile): one L2 prefetch per segment, also issued before the
      // dependency resolves, so that the CTA's whole weight share streams
      // from HBM while the previous kernel drains, and the stages after the
      // first S refill from L2.
      if constexpr (T::kPacked && MT == 1 && !T::kPair) {
        if (tiles_m == 1 && leader) {
          const uint64_t keep_w = l2_policy_evict_normal();
          SegIter it1;
          it1.init(p, me, ncta);
          Segment s1;
          int st_i = 0;
          while (it1.next(p, s1)) {
            const int nblk = s1.kb1 - s1.kb0;
            const int skip = min(nblk, max(0, pre - st_i));  // stages already loaded into the ring
            if (skip < nblk) {
              const uint8_t *src = p.packed + ((static_cast<int64_t>(s1.tile % p.tiles_n) * p.num_kb + s1.kb0 + skip) * KB) *
                                                  kPackedBlockBytes;
              bulk_prefetch_l2(src, static_cast<uint32_t>((nblk - skip) * KB * kPackedBlockBytes), keep_w);
            }
            st_i += nblk;
          }
        }
      }
      grid_dependency_wait();
      if constexpr (XQ != 0) {
        // the activation codes are written by this CTA's epilogue warps
        mbar_wait_warp(x_ready, 0u, p.status);
        __syncwarp();
        if (!staged) fence_proxy_async_global();
      }
      while (ok && it.next(p, sg)) {
        const int n0 = row0(sg.tile);
        const int m0 = (sg.tile / p.tiles_n) * BN;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++i) {
          const int s = i % S;
          const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
          uint8_t *st = smem + s * C::kStageBytes;
          if (i >= pre) {
            if (i >= S && !mbar_wait_warp(&empty[s], ph ^ 1u, p.status)) {
              ok = false;
              break;
            }
            if (leader && !staged) {
              if (!T::kPair || rank == 0)
                mbar_arrive_expect_tx(&full[s], T::kPair ? 2 * C::kTmaBytes : C::kTmaBytes);
              load_weights(st, &full[s], n0, kb);
            }
          }
          if (staged) {
            copy_x_rows(st, kb);
            if (leader) {
              if (i >= pre) {
                mbar_arrive_expect_tx(&full[s], C::kWBytes);
                load_weights(st, &full[s], n0, kb);
              } else {
                mbar_arrive(&full[s]);
              }
            }
          } else if (leader) {
            if constexpr (T::kPair) {
              // this CTA's half of the activation tile, 128 K per box
#pragma unroll
              for (int sub = 0; sub < C::kBSub; ++sub)
                tma_load_2d_pair(st + C::kBOff + sub * C::kBRows * 128, &tmB, mapa_shared(&full[s], 0u),
                                 kb * (T::kBRowBytes * KB / T::kBElemBytes) + sub * T::kBBoxElems,
                                 m0 + static_cast<int>(rank) * C::kBRows, keep_x);
            } else {
#pragma unroll
              for (int sub = 0; sub < C::kBSub; ++sub)
                tma_load_2d(st + C::kBOff + sub * BN * 128, &tmB, &full[s],
                            kb * (T::kBRowBytes * KB / T::kBElemBytes) + sub * T::kBBoxElems, m0, keep_x);
            }
          }
          __syncwarp();
        }
      }
      if constexpr (T::kPair) {
        // the even CTA's commits release this CTA's slots: wait for the last
        // ones, so that none lands after this CTA has left
        for (int k = i > S ? i - S : 0; ok && k < i; ++k)
          if (!mbar_wait_warp(&empty[k % S], static_cast<uint32_t>(k / S) & 1u, p.status)) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    {
      const bool leader = elect_one();
      constexpr uint32_t idesc = mma_idesc(T::kPair ? 256 : 128, BN, T::kFmt, T::kSparse, T::kDFmt);
      // metadata of row tile i: 4 TMEM columns after all accumulators
      const uint32_t e_tmem = tmem_base + NB * C::kAccCols;
      SegIter it;
      it.init(p, me, ncta);
      Segment sg;
      int i = 0, j = 0;
      bool ok = !T::kPair || rank == 0;  // pairs: the even CTA issues for both
      while (ok && it.next(p, sg)) {
        const int b = j % NB;
        const int r = j / NB;
        if (r >= 1 && !mbar_wait_warp(&tmem_empty[b], static_cast<uint32_t>(r - 1) & 1u, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * C::kAccCols;  // row tile rt at + rt * BN
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++i) {
          const int s = i % S;
          const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
          if (!mbar_wait_warp(&full[s], ph, p.status) ||
              (T::kMetaTransform && !mbar_wait_warp(&meta_ready[s], ph, p.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st_addr = smem_addr(smem + s * C::kStageBytes);
          const uint32_t b_addr = st_addr + C::kBOff;
          if (leader) {
            if (T::kSparse) {
              // 128 rows x 16 B, rows contiguous: core matrices of 8 rows are 128 B apart.
              if constexpr (T::kFp4) {
                // the two blocks' metadata boxes, 2048 bytes apart
                tmem_copy_128x256b(e_tmem, smem_desc(st_addr + C::kEOff, 128 * T::kERowBytes, 128, kSwizzleNone));
              } else if constexpr (T::kPair) {
                // each CTA's block metadata into its own tensor memory (two
                // blocks: the second 16-byte column is the next block's, 10240
                // bytes on)
                if constexpr (KB == 2)
                  tmem_copy_128x256b_pair(e_tmem, smem_desc(st_addr + C::e_off(0), kPackedBlockBytes, 128, kSwizzleNone));
                else
                  tmem_copy_128x128b_pair(e_tmem, smem_desc(st_addr + C::e_off(0), 2048, 128, kSwizzleNone));
              } else if constexpr (T::kPacked && MT * KB == 2) {
                // two packed blocks' metadata in one copy (both row tiles, or
                // both k-blocks of one row tile): the second 16-byte column is
                // the next block's metadata, 10240 bytes on
                tmem_copy_128x256b(e_tmem, smem_desc(st_addr + C::e_off(0), kPackedBlockBytes, 128, kSwizzleNone));
              } else {
#pragma unroll
                for (int rt = 0; rt < MT; ++rt) {
                  const uint32_t e_addr = st_addr + C::e_off(rt) + (T::kMetaTransform ? C::kEBytes : 0);
                  tmem_copy_128x128b(e_tmem + 4 * rt, smem_desc(e_addr, 2048, 128, kSwizzleNone));
                }
              }
            }
#pragma unroll
            for (int rt = 0; rt < MT; ++rt) {
              const uint32_t a_addr = st_addr + C::a_off(rt);
#pragma unroll
              for (int kk = 0; kk < C::kMmas; ++kk) {
                // MMA kk reads block kk / kMmas of the stage (packed blocks are
                // 10240 bytes apart), step kk % kMmas within it
                const uint32_t a_k = (KB == 1 || T::kFp4) ? kk * T::kAStep
                                                          : (kk / T::kMmas) * kPackedBlockBytes + (kk % T::kMmas) * T::kAStep;
                const uint64_t ad = smem_desc(a_addr + a_k, 16, T::kASbo, T::kASwizzle);
                const uint32_t boff = (kk * T::kBStep / 128) * (C::kBRows * 128) + (kk * T::kBStep) % 128;
                const uint64_t bd = smem_desc(b_addr + boff, 16, 8 * 128, kSwizzle128B);
                const uint32_t acc = (kb > sg.kb0 || kk > 0) ? 1u : 0u;
                const uint32_t d = d_tmem + rt * BN;
                if constexpr (T::kPair) {
                  mma_f8_sparse_pair(d, ad, bd, idesc, e_tmem + 2 * kk, acc);
                } else if constexpr (KIND == kSparseE4M3 || KIND == kSparseE4M3Packed || KIND == kSparseFP4) {
                  mma_f8_sparse(d, ad, bd, idesc, e_tmem + 4 * rt + 2 * kk, acc);
                } else if constexpr (KIND == kSparseI8Packed) {
                  mma_i8_sparse(d, ad, bd, idesc, e_tmem + 4 * rt + 2 * kk, acc);
                } else if constexpr (KIND == kSparseBF16) {
                  // one metadata column per MMA; columns are addressed in pairs and
                  // the instruction descriptor's selector picks the column of the pair
                  mma_bf16_sparse(d, ad, bd, idesc | static_cast<uint32_t>(kk & 1), e_tmem + (kk & ~1), acc);
                } else {
                  mma_f8_dense(d, ad, bd, idesc, acc);
                }
              }
            }
            if constexpr (T::kPair)
              mma_commit_pair(&empty[s], 3);  // both CTAs' slot
            else
              mma_commit(&empty[s]);
          }
          __syncwarp();
        }
        if (leader) {
          if constexpr (T::kPair)
            mma_commit_pair(&tmem_full[b], 3);
          else
            mma_commit(&tmem_full[b]);
        }
        __syncwarp();
        ++j;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue warps
    static_assert(XQ == 0 || C::kEpiWarps == 4, "the fused quantisation runs on four epilogue warps");
    const int e = warp - 2;          // epilogue warp index
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;   // W row within the tile == accumulator lane
    const int t = threadIdx.x - 64;  // 0 .. kEpiThreads - 1
    const int rt0 = (e >> 2) * C::kRtPerWarp;  // first row tile this warp drains
    float sx;
    if constexpr (XQ != 0)
      sx = fused_quantize<XQ>(p, t, s_xred, s_xscale, x_ready, C::kXStage > 0 && p.xstaged ? xstage : nullptr);
    else
      sx = p.x_scale ? __ldg(p.x_scale) : 1.0f;
    const float sw = p.w_scale ? __ldg(p.w_scale) : 1.0f;
    const float sc = sx * sw;
    constexpr int kW = C::kEpiCols;
    [[maybe_unused]] uint32_t ypass = 0;  // staged Y passes issued so far
    // accumulator b drained (pairs: the even CTA's MMA warp waits for both)
    auto release_acc = [&](int b) {
      if (T::kPair && rank != 0)
        mbar_arrive_cluster(mapa_shared(&tmem_empty[b], 0u));
      else
        mbar_arrive(&tmem_empty[b]);
    };
    SegIter it;
    it.init(p, me, ncta);
    Segment sg;
    int i = 0, j = 0;
    while (it.next(p, sg)) {
      if constexpr (T::kMetaTransform) {
        // Lane L = r0 + 8h + 16g of the TMEM metadata holds, for each of the
        // stage's 4 MMAs, the 16 bits of K-half h of row 16g + r0 (low half)
        // and of row 16g + 8 + r0 (high half).
        const int r0 = t & 7, h = (t >> 3) & 1, g = t >> 4;
        const int ra = 16 * g + r0, rb = ra + 8;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++i) {
          const int s = i % S;
          const uint32_t ph = static_cast<uint32_t>(i / S) & 1u;
          if (!mbar_wait(&full[s], ph, p.status)) break;
          const uint8_t *e = smem + s * C::kStageBytes + C::kEOff;
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
      const int b = j % NB;
      const int r = j / NB;
      // fp32 partial tile of CTA g, row tile rt, in quads of 4 token columns
      // laid out [column quad][row][4], so that a warp's 32 rows of one quad
      // are 512 contiguous bytes: quad cq of this thread's row.
      // (g: schedule index; pairs keep one partial per CTA, 2 g + rank)
      auto part4 = [&](int g, int rt, int cq) {
        const int slot = T::kPair ? 2 * g + static_cast<int>(rank) : g;
        return reinterpret_cast<float4 *>(p.partials) +
               ((static_cast<size_t>(slot) * MT + rt) * (BN / 4) + cq) * 128 + row;
      };
      // the split tile's counter (pairs: one per CTA of the pair, counting
      // the contributors' CTAs of the same rank)
      const int ci = (sg.tile - p.dp_tiles) * (T::kPair ? 2 : 1) + static_cast<int>(rank);
      // Owner of a split tile: its contributors (the next CTAs) compute this
      // tile's later k-blocks as the first segment of their range, so they
      // are normally done before this CTA's own k-blocks are.  Wait for them
      // and (decode-sized tiles, where the tail matters) start loading the
      // first contributor's first pass before the accumulator is ready, so
      // that the L2 round trip overlaps the last MMAs instead of following
      // them.  Wide tiles load it after the accumulator wait: keeping the
      // registers live through their epilogue would spill.
      static_assert(C::kRtPerWarp == 1, "each epilogue warp drains one row tile");
      int first = 0, last = -1;  // contributor CTAs of an owned tile
      float4 nxt[8];             // the next pass's first-contributor partial
      if (sg.role == kOwner) {
        const int64_t u_first = static_cast<int64_t>(sg.tile - p.dp_tiles) * p.num_kb;
        first = me + 1;
        last = cta_of_unit(u_first + p.num_kb - 1, p.sk_units, p.sk_grid);
        if (t == 0) {
          const uint32_t expect = static_cast<uint32_t>(last - first + 1);
          const uint64_t t0 = global_timer_ns();
          uint32_t polls = 0;
          while (ld_acquire_gpu(&p.counters[ci]) < expect) {
            __nanosleep(20);
            if ((++polls & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
              if (p.status) atomicOr(p.status, SP24_STATUS_TIMEOUT);
              break;
            }
          }
          p.counters[ci] = 0u;  // leave the workspace counters at zero
        }
        named_bar_sync(1, C::kEpiThreads);  // the acquire by thread 0 covers the whole CTA's reads
        if constexpr (!C::kTmaStoreY) {
#pragma unroll
          for (int k4 = 0; k4 < kW / 4; ++k4) nxt[k4] = __ldcg(part4(first, rt0, k4));
        }
      }
      mbar_wait(&tmem_full[b], static_cast<uint32_t>(r) & 1u, p.status);
      tc_fence_after();
      const int n0 = row0(sg.tile);
      const int m0 = (sg.tile / p.tiles_n) * BN;
      const int mvalid = min(BN, p.M - m0);
      // lane quarter of this warp, accumulator b; row tile rt at + rt * BN
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * C::kAccCols;

      if (sg.role == kContrib) {
        // leave the fp32 partial tile (valid token columns) for the owner
#pragma unroll 1
        for (int rt = rt0; rt < rt0 + C::kRtPerWarp; ++rt) {
#pragma unroll 1
          for (int c = 0; c < mvalid; c += 16) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_acc + rt * BN + c, v);
            tmem_ld_wait();
            tmem_regs_ready(v);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              __stcg(part4(me, rt, c / 4 + k4),
                     make_float4(acc_f32<KIND>(v[4 * k4]), acc_f32<KIND>(v[4 * k4 + 1]),
                                 acc_f32<KIND>(v[4 * k4 + 2]), acc_f32<KIND>(v[4 * k4 + 3])));
          }
        }
        tc_fence_before();
        release_acc(b);
        // The barrier orders every thread's partial stores before thread 0's
        // release increment (release is cumulative), which the owner acquires.
        named_bar_sync(1, C::kEpiThreads);
        if (t == 0) red_release_add_gpu(&p.counters[ci], 1u);
      } else {
#pragma unroll 1
        for (int rt = rt0; rt < rt0 + C::kRtPerWarp; ++rt) {
          const int n = n0 + rt * 128 + row;
          // VS: y = acc * sx[m] * sw[n]; this thread's W row n has one sw,
          // and the pass's token scales are held one per lane (token_scale)
          // and shuffled to every lane.
          [[maybe_unused]] float swn = 0.0f;
          if constexpr (VS) swn = p.w_vec ? __ldg(p.w_scale + n) : sw;
          const uint32_t t_row = t_acc + rt * BN;
          // kW token columns per pass.  The first contributor's partial for
          // the next pass is loaded while this pass is summed and stored (for
          // the first pass of a narrow tile: before the accumulator was
          // ready, above), so an owned tile costs about one L2 round trip,
          // not one per pass.
          if constexpr (C::kTmaStoreY) {
            if (first <= last) {
#pragma unroll
              for (int k4 = 0; k4 < kW / 4; ++k4) nxt[k4] = __ldcg(part4(first, rt, k4));
            }
          }
          // Y through shared memory: this warp's 32 rows of one 32-token pass
          // (see Config), staged token-major as rows of Y.  Lane 0 issues the
          // warp's stores; before a buffer is rewritten it waits until the
          // store issued from it two passes ago has read it.
          auto store_pass = [&](int c, auto &&value_of) {
            uint16_t *buf = reinterpret_cast<uint16_t *>(ystage + (e * 2 + (ypass & 1)) * C::kStageY);
            [[maybe_unused]] float xs = 0.0f;
            if constexpr (VS) xs = token_scale(p, m0 + c + lane, sx);
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 32; k += 2) {  // two tokens per conversion
              float f0 = sc, f1 = sc;
              if constexpr (VS) {
                f0 = __shfl_sync(0xFFFFFFFFu, xs, k) * swn;
                f1 = __shfl_sync(0xFFFFFFFFu, xs, k + 1) * swn;
              }
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(value_of(k) * f0, value_of(k + 1) * f1);
              buf[k * 32 + lane] = __bfloat16_as_ushort(h2.x);
              buf[(k + 1) * 32 + lane] = __bfloat16_as_ushort(h2.y);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, buf, n0 + rt * 128 + q * 32, m0 + c);
              bulk_commit_group();
            }
            ++ypass;
          };
          if constexpr (C::kTmaStoreY) {
            if (first > last) {
              // Whole tile: up to 128 accumulator columns per TMEM wait (the
              // wait, not the arithmetic, dominates a pass), stored as 32-token
              // passes.  Tokens past M fall outside the tensor map.
              // (64 columns per wait with scale vectors, for register room)
              constexpr int kStep = VS ? 64 : 128;
#pragma unroll 1
              for (int c2 = 0; c2 < mvalid; c2 += kStep) {
                uint32_t w0[64], w1[64];
                tmem_ld_32x32b_x64(t_row + c2, w0);
                if (!VS && c2 + 64 < BN) tmem_ld_32x32b_x64(t_row + c2 + 64, w1);
                tmem_ld_wait();
                tmem_regs_ready(w0);
                if constexpr (!VS) tmem_regs_ready(w1);
#pragma unroll
                for (int h = 0; h < kStep / 32; ++h) {
                  if (c2 + 32 * h < mvalid)
                    store_pass(c2 + 32 * h, [&](int k) {
                      return acc_f32<KIND>(h < 2 ? w0[32 * h + k] : w1[32 * (h - 2) + k]);
                    });
                }
              }
              continue;
            }
          }
#pragma unroll 1
          for (int c = 0; c < mvalid; c += kW) {
            uint32_t v[2][16];
            tmem_ld_32x32b_x16(t_row + c, v[0]);
            if constexpr (kW == 32) tmem_ld_32x32b_x16(t_row + c + 16, v[1]);
            tmem_ld_wait();
            tmem_regs_ready(v[0]);
            tmem_regs_ready(v[1]);
            float acc[32];
#pragma unroll
            for (int k = 0; k < kW; ++k) acc[k] = acc_f32<KIND>(v[k >> 4][k & 15]);
            if (first <= last) {
              float4 cur[8];
#pragma unroll
              for (int k4 = 0; k4 < kW / 4; ++k4) cur[k4] = nxt[k4];
              if (c + kW < mvalid) {
#pragma unroll
                for (int k4 = 0; k4 < kW / 4; ++k4) nxt[k4] = __ldcg(part4(first, rt, (c + kW) / 4 + k4));
              }
#pragma unroll
              for (int k4 = 0; k4 < kW / 4; ++k4) {
                acc[4 * k4] += cur[k4].x;
                acc[4 * k4 + 1] += cur[k4].y;
                acc[4 * k4 + 2] += cur[k4].z;
                acc[4 * k4 + 3] += cur[k4].w;
              }
              for (int g2 = first + 1; g2 <= last; ++g2) {  // further contributors, in CTA order
                float4 pv[8];
#pragma unroll
                for (int k4 = 0; k4 < kW / 4; ++k4) pv[k4] = __ldcg(part4(g2, rt, c / 4 + k4));
#pragma unroll
                for (int k4 = 0; k4 < kW / 4; ++k4) {
                  acc[4 * k4] += pv[k4].x;
                  acc[4 * k4 + 1] += pv[k4].y;
                  acc[4 * k4 + 2] += pv[k4].z;
                  acc[4 * k4 + 3] += pv[k4].w;
                }
              }
            }
            if constexpr (C::kTmaStoreY) {
              // Stage the pass token-major, as rows of Y (32 tokens x 128 W
              // rows), and store it with one bulk tensor copy.
              store_pass(c, [&](int k) { return acc[k]; });
            } else {
              [[maybe_unused]] float xs = 0.0f;
              if constexpr (VS) xs = token_scale(p, m0 + c + lane, sx);
#pragma unroll
              for (int k = 0; k < kW; ++k) {
                const int m = m0 + c + k;
                float f = sc;
                if constexpr (VS) f = __shfl_sync(0xFFFFFFFFu, xs, k) * swn;
                if (m < p.M) p.y[static_cast<size_t>(m) * p.N + n] = f32_to_bf16_bits(acc[k] * f);
              }
            }
          }
        }
        tc_fence_before();
        release_acc(b);
      }
      ++j;
    }
    if constexpr (C::kTmaStoreY) {
      if (lane == 0) bulk_wait_group_all();  // Y written before the CTA leaves
    }
  }

  tc_fence_before();
  __syncthreads();
  // pairs: no CTA frees its tensor memory or leaves while the other may still
  // use it, arrive on its barriers or load into its shared memory
  if constexpr (T::kPair) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (T::kPair)
      tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else
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

// Row-major 2-D map: `inner` elements per row (contiguous), `outer` rows;
// elem_bytes = 0 marks 4-bit elements (two per byte).
bool make_tensor_map_2d(CUtensorMap *map, const void *ptr, CUtensorMapDataType dt, int elem_bytes,
                        uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {elem_bytes == 0 ? inner / 2 : inner * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token-tile width: the MMA N.  Small token counts use the smallest tile
// that holds them; medium ones 128 (two accumulators); large ones prefer 224
// (still two accumulators, so epilogues overlap main loops) unless it pads
// more than 10% over 256.
static int choose_bn(GemmKind kind, int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M < 1024 || kind == kSparseBF16) return 128;
  const long pad224 = static_cast<long>((M + 223) / 224) * 224;
  return pad224 * 10 <= static_cast<long>(M) * 11 ? 224 : 256;
}

// Clusters of two CTAs of the SM-pair GEMM that the device runs at once (0
// when it cannot run them: no device, or no room for a pair).
static int pair_capacity() {
  static int cap = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    using C = Config<kSparseE4M3Pair, 224, 1, 1, 0>;
    const auto kern = gemm_kernel<kSparseE4M3Pair, 224, 1, 0, 1, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess) {
      (void)cudaGetLastError();
      return;
    }
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(2, 1, 1);
    qc.blockDim = dim3(C::kThreads, 1, 1);
    qc.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.attrs = qa;
    qc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &qc) == cudaSuccess)
      cap = n;
    else
      (void)cudaGetLastError();
  });
  return cap;
}

GemmPlan plan_gemm(GemmKind kind, int M, int N, int K, int sm_count) {
  GemmPlan pl{};
  const bool pair = kind == kSparseE4M3Pair;
  pl.bn = choose_bn(kind, M);
  // Large token tiles (224 tokens: many tiles, bound by operand ingest) pair
  // two 128-row W tiles on one activation tile when N allows it.
  pl.mt = (pl.bn == 224 && kind != kSparseBF16 && N % 256 == 0) ? 2 : 1;
  // Decode-sized tiles over packed weights take two 128-K blocks per stage;
  // FP4 always does (one 4-bit box spans two blocks) and uses one row tile.
  // SM pairs: each CTA one row tile of a 256-row tile, scheduled by pair.
  if (kind == kSparseFP4 || pair) pl.mt = 1;
  if (pair) sm_count = min(sm_count / 2, pair_capacity());
  pl.kb = (kind == kSparseFP4 || (pair && K % 256 == 0) ||
           ((kind == kSparseE4M3Packed || kind == kSparseI8Packed) && pl.bn <= 64 && pl.mt == 1 && K % 256 == 0))
              ? 2
              : 1;
  pl.bk = 128 * pl.kb;
  pl.tiles_n = N / (pair ? 256 : 128 * pl.mt);
  pl.tiles_m = (M + pl.bn - 1) / pl.bn;
  pl.num_kb = K / pl.bk;
  pl.num_tiles = pl.tiles_n * pl.tiles_m;
  pl.units = static_cast<int64_t>(pl.num_tiles) * pl.num_kb;
  // Persistent grid: one CTA per SM, fewer only when there are fewer than
  // two k-blocks per CTA.
  int64_t G = pl.units / 2;
  if (G > sm_count) G = sm_count;
  if (G < 1) G = 1;
  pl.grid = static_cast<int>(G);
  // Whole tiles for the full waves, stream-K over the leftover tiles so that
  // the last partial wave is spread over every CTA.
  pl.dp_tiles = (pl.num_tiles / pl.grid) * pl.grid;
  const int rem = pl.num_tiles - pl.dp_tiles;
  pl.sk_units = static_cast<int64_t>(rem) * pl.num_kb;
  // Tiles wider than 64 tokens are split at most two ways: their owners then
  // read a single, prefetched partial.  Narrower (decode) tiles have at most
  // two epilogue passes, so they split as finely as the grid allows.
  int64_t skg = pl.sk_units / 2;  // at least two k-blocks per CTA
  if (skg > pl.grid) skg = pl.grid;
  if (pl.bn > 64 && skg > 2 * static_cast<int64_t>(rem)) skg = 2 * static_cast<int64_t>(rem);
  if (skg < rem) skg = rem;
  pl.sk_grid = rem > 0 ? static_cast<int>(skg) : 0;
  if (pl.dp_tiles == 0) pl.grid = pl.sk_grid;  // no idle CTAs when every tile is split
  pl.stream_k = rem > 0;
  pl.counter_bytes = pl.stream_k ? kGemmCounterBytes : 0;
  pl.partial_bytes =
      pl.stream_k ? static_cast<size_t>(pl.sk_grid) * 128 * pl.mt * pl.bn * sizeof(float) : 0;
  if (pair) {  // the schedule counted pairs; launch and partials count CTAs
    pl.grid *= 2;
    pl.partial_bytes *= 2;
  }
  pl.pair = pair ? 1 : 0;
  return pl;
}

GemmKind packed_kind(int M, int N, int K, int sm_count) {
  const GemmPlan pl = plan_gemm(kSparseE4M3Packed, M, N, K, sm_count);
  const bool wide = pl.mt == 2 && pl.bn == 224;                      // prefill-sized
  const bool mid = pl.bn == 128 && M > 128 && N % 256 == 0;          // several 128-token tiles
  return ((wide || mid) && pair_capacity() >= 2) ? kSparseE4M3Pair : kSparseE4M3Packed;
}

template <int KIND, int BN, int MT, int XQ = 0, int KB = 1, bool VS = false>
static cudaError_t launch_typed(const GemmPlan &pl, const void *xq, const float *x_scale,
                                const void *w_values, const uint8_t *w_meta, const float *w_scale,
                                void *y, int M, int N, int K, void *workspace, int32_t *status,
                                cudaStream_t st, const GemmFusedX *fx = nullptr, int x_vec = 0,
                                int w_vec = 0) {
  using T = KindTraits<KIND>;
  using C = Config<KIND, BN, MT, KB, XQ>;
  static_assert(XQ == 0 || KIND == kSparseE4M3Packed, "fused quantisation feeds the packed E4M3 GEMM");
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(gemm_kernel<KIND, BN, MT, XQ, KB, VS>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;

  CUtensorMap tmA, tmB, tmE;
  const CUtensorMapDataType dtA = T::kFp4                 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B
                                  : T::kAElemBytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapDataType dtB = T::kFp4                 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B
                                  : T::kBElemBytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint64_t a_row = T::kSparse ? static_cast<uint64_t>(K) / 2 : static_cast<uint64_t>(K);
  const CUtensorMapSwizzle a_sw =
      T::kASwizzle == kSwizzle64B ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (T::kPair) {
    // the packed buffer as rows of 256 bytes: a 10240-byte block is 40 rows
    const uint64_t packed_bytes = static_cast<uint64_t>(N) * K / 2 + static_cast<uint64_t>(N) * K / 8;
    if (!make_tensor_map_2d(&tmA, w_values, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, packed_bytes / 256, 256,
                            KB * kPackedBlockBytes / 256, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else if (T::kPacked) {
    tmA = {};
  } else if (T::kFp4) {
    // the stored codes of 128 rows x 256 K: one 128-element 4-bit box
    if (!make_tensor_map_2d(&tmA, w_values, dtA, 0, a_row, N, 128, C::kRows, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else if (!make_tensor_map_2d(&tmA, w_values, dtA, T::kAElemBytes, a_row, N,
                                 T::kARowBytes / T::kAElemBytes, C::kRows, a_sw)) {
    return cudaErrorInvalidValue;
  }
  if (!make_tensor_map_2d(&tmB, xq, dtB, T::kFp4 ? 0 : T::kBElemBytes, K, M, T::kBBoxElems, C::kBRows,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (T::kSparse && !T::kPacked) {
    if (!make_tensor_map_2d(&tmE, w_meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(K) / 8, N,
                            16, C::kRows, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    tmE = tmB;  // unused
  }
  if (T::kPacked && !T::kPair) tmA = tmB;  // unused
  CUtensorMap tmY = tmB;       // unused unless Y is stored through shared memory
  if (C::kTmaStoreY &&
      !make_tensor_map_2d(&tmY, y, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, N, M, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.num_kb = pl.num_kb;
  a.tiles_n = pl.tiles_n;
  a.num_tiles = pl.num_tiles;
  a.dp_tiles = pl.dp_tiles;
  a.sk_grid = pl.sk_grid;
  a.sk_units = pl.sk_units;
  a.y = static_cast<uint16_t *>(y);
  a.x_scale = x_scale;
  a.w_scale = w_scale;
  // Workspace layout: tile counters in a fixed-size prefix (zero between
  // calls, whatever the shape), then the fp32 partial tiles (scratch).
  a.counters = pl.stream_k ? static_cast<uint32_t *>(workspace) : nullptr;
  a.partials = pl.stream_k
                   ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kGemmCounterBytes)
                   : nullptr;
  a.status = status;
  a.packed = T::kPacked ? static_cast<const uint8_t *>(w_values) : nullptr;
  a.x = nullptr;
  a.xq = nullptr;
  a.x_scale_out = nullptr;
  a.xvec = 0;
  a.xstaged = 0;
  a.x_vec = x_vec;
  a.w_vec = w_vec;
  if constexpr (XQ != 0) {
    a.x = static_cast<const uint16_t *>(fx->x);
    a.xq = fx->xq;
    a.x_scale_out = fx->x_scale;
    a.xvec = static_cast<int64_t>(M) * (XQ == 2 ? K / 3 * 2 : K) / 8;
    if (a.xvec > kFusedXVec) return cudaErrorInvalidValue;
    a.xstaged = (C::kXStage > 0 && static_cast<int64_t>(M) * K <= kXStageBytes) ? 1 : 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  // Programmatic dependent launch (see the kernel).  Stream-K owners wait
  // for contributor CTAs, which only needs every CTA to become resident
  // eventually: the grid is at most one CTA per SM, so every CTA is resident
  // as soon as the kernels ahead of it drain, and each wait is bounded
  // anyway.  The launch is not cooperative: a cooperative grid was measured
  // to start 1-2 us later behind the previous kernel, losing the weight
  // prefetch that programmatic launch overlaps with it.
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  attrs[1].id = cudaLaunchAttributeClusterDimension;  // SM pairs: clusters of two
  attrs[1].val.clusterDim.x = 2;
  attrs[1].val.clusterDim.y = 1;
  attrs[1].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = T::kPair ? 2 : 1;
  if (T::kPair && pl.grid % 2 != 0) return cudaErrorInvalidValue;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<KIND, BN, MT, XQ, KB, VS>, tmA, tmB, tmE, tmY, a);
}

template <int KIND>
static cudaError_t launch_kind(const GemmPlan &pl, const void *xq, const float *x_scale,
                               const void *w_values, const uint8_t *w_meta, const float *w_scale,
                               void *y, int M, int N, int K, void *ws, int32_t *status,
                               cudaStream_t st) {
  if constexpr (KIND == kSparseE4M3Pair) {
    if (pl.bn == 224 && pl.kb == 2)
      return launch_typed<KIND, 224, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    if (pl.bn == 224)
      return launch_typed<KIND, 224, 1, 0, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    if (pl.bn == 128 && pl.kb == 2)
      return launch_typed<KIND, 128, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    if (pl.bn == 128)
      return launch_typed<KIND, 128, 1, 0, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
    return cudaErrorInvalidValue;
  } else if constexpr (KIND == kSparseFP4) {
    switch (pl.bn) {
      case 16: return launch_typed<KIND, 16, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 32: return launch_typed<KIND, 32, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 64: return launch_typed<KIND, 64, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 128: return launch_typed<KIND, 128, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 224: return launch_typed<KIND, 224, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 256: return launch_typed<KIND, 256, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      default: return cudaErrorInvalidValue;
    }
  } else {
    if constexpr (KIND == kSparseE4M3Packed || KIND == kSparseI8Packed) {
      if (pl.kb == 2) {
        switch (pl.bn) {
          case 16: return launch_typed<KIND, 16, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
          case 32: return launch_typed<KIND, 32, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
          case 64: return launch_typed<KIND, 64, 1, 0, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
          default: return cudaErrorInvalidValue;
        }
      }
    }
    switch (pl.bn) {
      case 16: return launch_typed<KIND, 16, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 32: return launch_typed<KIND, 32, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 64: return launch_typed<KIND, 64, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 128: return launch_typed<KIND, 128, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 224:
        if constexpr (KIND != kSparseBF16) {
          if (pl.mt == 2)
            return launch_typed<KIND, 224, 2>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
        }
        return launch_typed<KIND, 224, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      case 256: return launch_typed<KIND, 256, 1>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, ws, status, st);
      default: return cudaErrorInvalidValue;
    }
  }
}

template <int XQ>
static cudaError_t launch_quant_bn(const GemmPlan &pl, const GemmFusedX &fx, const void *packed,
                                   const float *w_scale, void *y, int M, int N, int K, void *ws,
                                   int32_t *status, cudaStream_t st) {
  constexpr int P = kSparseE4M3Packed;
  if (pl.kb == 2) {
    switch (pl.bn) {
      case 16: return launch_typed<P, 16, 1, XQ, 2>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
      case 32: return launch_typed<P, 32, 1, XQ, 2>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
      case 64: return launch_typed<P, 64, 1, XQ, 2>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (pl.bn) {
    case 16: return launch_typed<P, 16, 1, XQ>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
    case 32: return launch_typed<P, 32, 1, XQ>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
    case 64: return launch_typed<P, 64, 1, XQ>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
    case 128: return launch_typed<P, 128, 1, XQ>(pl, fx.xq, nullptr, packed, nullptr, w_scale, y, M, N, K, ws, status, st, &fx);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm_scaled(const GemmPlan &pl, const void *xq, const float *x_scales, int x_vec,
                               const void *packed, const float *w_scales, int w_vec, void *y, int M, int N,
                               int K, void *ws, int32_t *status, cudaStream_t st) {
  constexpr int P = kSparseE4M3Packed;
  if (pl.pair) {
#define SP24_SCALED_PAIR(BN_, KB_)                                                                            \
  return launch_typed<kSparseE4M3Pair, BN_, 1, 0, KB_, true>(pl, xq, x_scales, packed, nullptr, w_scales, y, M, N, \
                                                             K, ws, status, st, nullptr, x_vec, w_vec)
    if (pl.bn == 224 && pl.kb == 2) SP24_SCALED_PAIR(224, 2);
    if (pl.bn == 224) SP24_SCALED_PAIR(224, 1);
    if (pl.bn == 128 && pl.kb == 2) SP24_SCALED_PAIR(128, 2);
    if (pl.bn == 128) SP24_SCALED_PAIR(128, 1);
#undef SP24_SCALED_PAIR
    return cudaErrorInvalidValue;
  }
#define SP24_SCALED(BN_, MT_, KB_)                                                                        \
  return launch_typed<P, BN_, MT_, 0, KB_, true>(pl, xq, x_scales, packed, nullptr, w_scales, y, M, N, K, ws, \
                                                 status, st, nullptr, x_vec, w_vec)
  if (pl.kb == 2) {
    switch (pl.bn) {
      case 16: SP24_SCALED(16, 1, 2);
      case 32: SP24_SCALED(32, 1, 2);
      case 64: SP24_SCALED(64, 1, 2);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (pl.bn) {
    case 16: SP24_SCALED(16, 1, 1);
    case 32: SP24_SCALED(32, 1, 1);
    case 64: SP24_SCALED(64, 1, 1);
    case 128: SP24_SCALED(128, 1, 1);
    case 224:
      if (pl.mt == 2) SP24_SCALED(224, 2, 1);
      SP24_SCALED(224, 1, 1);
    case 256: SP24_SCALED(256, 1, 1);
    default: return cudaErrorInvalidValue;
  }
#undef SP24_SCALED
}

cudaError_t launch_gemm_quant(const GemmPlan &pl, const GemmFusedX &fx, const void *packed,
                              const float *w_scale, void *y, int M, int N, int K, void *workspace,
                              int32_t *status, cudaStream_t st) {
  if (pl.mt != 1) return cudaErrorInvalidValue;
  return fx.lift ? launch_quant_bn<2>(pl, fx, packed, w_scale, y, M, N, K, workspace, status, st)
                 : launch_quant_bn<1>(pl, fx, packed, w_scale, y, M, N, K, workspace, status, st);
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
    case kSparseE4M3Packed:
      return launch_kind<kSparseE4M3Packed>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    case kSparseI8Packed:
      return launch_kind<kSparseI8Packed>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    case kSparseFP4:
      return launch_kind<kSparseFP4>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    case kSparseE4M3Pair:
      return launch_kind<kSparseE4M3Pair>(pl, xq, x_scale, w_values, w_meta, w_scale, y, M, N, K, workspace, status, st);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace sp24
