// stream.cu -- the bandwidth-bound steps of the path as single-launch,
// TMA-streamed kernels:
//   kOpQuantize  per-tensor E4M3 quantisation of activations,
//   kOpLift      the same fused with the 6:8 activation lift,
//   kOpPrune24   2:4 magnitude prune + quantise + compress of weights,
//   kOpPrune24Packed  the same, written in the GEMM's tile-packed layout,
//   kOpSlide68   6:8 prune + sliding-window decomposition of weights,
//   kOpSlide68Packed  the same, written in the GEMM's tile-packed layout.
//
// One CTA per SM (cooperative launch: all CTAs resident), each owning a
// contiguous range of 32 KB chunks of the bf16 input (for the packed 2:4 op a
// chunk is the 128 x 128 box of W behind one packed block, read with a 2-D
// tensor copy).  A producer warp streams the chunks into a 5-stage
// shared-memory ring (full/empty mbarriers per slot), 16 consumer warps work
// on interleaved 16-byte units of each chunk.
//   Phase 1: amax of the slice, and for the prune ops the group selection,
//            whose metadata goes straight to global memory (this phase is
//            bound by HBM, so the selection's arithmetic hides under it).
//   Grid barrier: the CTAs combine their amax through device counters that
//            the last CTA to leave resets; every CTA derives s = amax / 448
//            and fills a 64 KB table in shared memory with the E4M3 code of
//            every bf16 bit pattern: the 24 binades below amax computed as
//            the definition states, E4M3(RN_fp32(x / s)), signed zeros for
//            everything smaller.
//   Phase 2: codes by table lookup (2:4: of the kept pair named by the
//            metadata, read back one chunk ahead); the slice comes from the
//            ring again when the CTA's whole range fitted in it, else it is
//            re-streamed in reverse chunk order, so the chunks phase 1 read
//            last, the likeliest to still be in L2, are read first.
// The bf16-output prune ops need no scale and finish after phase 1.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

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
constexpr int kStages = 5;
constexpr int kTab = 24 * 128;               // binades x mantissas that can give a nonzero code
constexpr int kTabBytes = 65536;             // code of every bf16 bit pattern
// SMALL instantiations serve tensors of at most 2 chunks per CTA: they keep
// the whole slice resident in a 2-slot ring and divide directly, so they need
// no table and little shared memory (which leaves room on the SM for the
// next kernel's CTAs to start early).
template <bool SMALL> __host__ __device__ constexpr int ring_stages() { return SMALL ? 2 : kStages; }
template <bool SMALL> __host__ __device__ constexpr int table_bytes() { return SMALL ? 0 : kTabBytes; }
template <bool SMALL>
constexpr uint32_t smem_bytes() {
  return ring_stages<SMALL>() * kChunkBytes + table_bytes<SMALL>() + 2 * ring_stages<SMALL>() * 8 + 128;
}
static_assert(smem_bytes<false>() + 2048 <= 227 * 1024, "ring + table exceed the shared memory of a CTA");

enum StreamOp : int {
  kOpQuantize = 0,
  kOpLift = 1,
  kOpPrune24 = 2,
  kOpSlide68 = 3,
  kOpPrune24Packed = 4,
  kOpSlide68Packed = 5
};

// Bytes of input one consumer thread handles as one unit: 8 bf16 (one
// metadata byte of 2:4, one 8-group of the lift) or 16 bf16 for 6:8 (two
// 8-groups = three metadata bytes).  Unit r of thread t in a chunk starts at
// byte r * kConsumers * kUnit + t * kUnit: consecutive threads read
// consecutive 16-byte words (no shared-memory bank conflicts) and write
// consecutive outputs.
template <int OP>
__host__ __device__ constexpr int unit_bytes() { return OP == kOpSlide68 || OP == kOpSlide68Packed ? 32 : 16; }

struct StreamArgs {
  // The packed ops read W through this 2-D map.  kOpPrune24Packed: box 128
  // rows x 128 bf16, chunk c is the input of packed block c (rows
  // 128 (c / kblocks) .., columns 128 (c % kblocks) ..).  kOpSlide68Packed:
  // box 64 rows x 256 bf16 = the input of rows 64 h .. of packed blocks
  // 3 kg .. 3 kg + 2 of row tile t, for chunk c = (t K/256 + kg) 2 + h.
  CUtensorMap wmap;
  const uint8_t *x;  // bf16 input
  int64_t nbytes;    // input bytes, a multiple of 32
  int64_t nchunks;
  uint32_t *ws;      // [0] amax bits, [1] arrivals, [2] departures
  float *scale_out;
  int32_t *status;
  uint8_t *out;      // codes / kept values (the packed blocks for kOpPrune24Packed)
  uint8_t *meta;
  uint8_t *dense;
  uint32_t kblocks;  // packed ops: K-blocks of the compressed operand per row (K / 128, 6:8: K' / 128)
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void red_max_relaxed_gpu(uint32_t *p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_add_release_gpu(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// E4M3 code of a bf16 pattern by lookup: entry h of the 64 KB table is the
// code of the bf16 pattern h.  Only the 24 binades at and below amax's can
// give a nonzero code (smaller magnitudes are below 2^-13 after division);
// every other pattern holds the zero code of its sign.  DIRECT (tensors too
// small to amortise the table) computes the code by the same division.
template <bool DIRECT>
struct CodeTable {
  const uint8_t *tab;
  float s;
  __device__ __forceinline__ uint32_t operator()(uint32_t h) const {
    if constexpr (DIRECT)
      return e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s));
    else
      return tab[h];
  }
  // codes of the bf16 values h0 (elements 0, 1) and h1 (2, 3), byte i = element i
  __device__ __forceinline__ uint32_t codes4(uint32_t h0, uint32_t h1) const {
    return (*this)(h0 & 0xFFFFu) | (*this)(h0 >> 16) << 8 | (*this)(h1 & 0xFFFFu) << 16 | (*this)(h1 >> 16) << 24;
  }
};

// The same codes without a table: q = RN(x * RN(1 / s)) and the codes 8
// steps either side of it, four values at once (e4m3_codes4_quot); the
// correctly rounded division where that cannot decide (about one value in
// 2^16).  Cheaper per code than the byte lookups of the table, which conflict
// on shared-memory banks.
struct CodeQuot {
  float s, r;
  __device__ __forceinline__ uint32_t operator()(uint32_t h) const {
    return e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s));
  }
  __device__ __forceinline__ uint32_t codes4(uint32_t h0, uint32_t h1) const {
    uint32_t q;
    if (!e4m3_codes4_quot(h0, h1, r, q)) q = e4m3_codes4_div(h0, h1, s);
    return q;
  }
};

// Every E4M3 op encodes with CodeQuot except the unpacked 2:4 prune that also
// writes the pruned dense copy (one code per kept element, from the table).
template <int OP, bool DENSE>
__host__ __device__ constexpr bool quot_encoder() {
  return !(OP == kOpPrune24 && DENSE);
}

// The table: signed zeros everywhere (zero_table, before phase 1), then the
// 24 binades below amax (fill_table), each entry as the definition states,
// E4M3(RN_fp32(x / s)) (the code of -x is the code of x with the sign bit).
__device__ __forceinline__ void zero_table(uint8_t *tab, int t) {
  uint4 *t4 = reinterpret_cast<uint4 *>(tab);
  for (int i = t; i < kTabBytes / 16; i += kConsumers) {
    const uint32_t z = i < kTabBytes / 32 ? 0u : 0x80808080u;
    t4[i] = make_uint4(z, z, z, z);
  }
}

__device__ __forceinline__ void fill_table(uint8_t *tab, uint32_t amax_bits, float s, int t) {
  const int e_base = static_cast<int>(amax_bits >> 7) - 23;
  for (int i = t; i < kTab; i += kConsumers) {
    const int e = e_base + i / 128;
    if (e >= 0 && e < 255) {
      const uint32_t h = (static_cast<uint32_t>(e) << 7) | static_cast<uint32_t>(i & 127);
      const uint32_t c = e4m3_code(__fdiv_rn(bf16_bits_to_float(h), s)) & 0x7Fu;
      tab[h] = static_cast<uint8_t>(c);
      tab[h | 0x8000u] = static_cast<uint8_t>(c | 0x80u);
    }
  }
}

__device__ __forceinline__ void halves(const uint4 v, uint32_t h[8]) {
  h[0] = v.x & 0xFFFFu; h[1] = v.x >> 16; h[2] = v.y & 0xFFFFu; h[3] = v.y >> 16;
  h[4] = v.z & 0xFFFFu; h[5] = v.z >> 16; h[6] = v.w & 0xFFFFu; h[7] = v.w >> 16;
}

// A chunk's first element e (a multiple of kChunkBytes / 2).  Unit u of the
// chunk starts at element e + u * kUnit / 2; addresses are formed as
// per-chunk 64-bit bases plus 32-bit offsets of u.
struct Chunk {
  uint64_t e;
  uint64_t idx;     // the chunk's index (= its packed block for kOpPrune24Packed)
  uint8_t *group;   // kOpSlide68Packed: packed block (t, 3 kg) of the chunk
  uint32_t row0;    // kOpSlide68Packed: first row in the row tile (0 or 64)
};

// ------------------------------------------------------------------ 2:4 + E4M3
// The 2:4 selection and E4M3 codes of one 8-element unit (two groups), from
// its four 32-bit words (two bf16 each, lower index in the low half).
// Every element gets the key  |w| << 17 | (3 - i) << 1 | sign:  keys are
// unique, and "larger key" is exactly "beats" of the rule (larger |w|, or
// equal |w| at the lower index), so the kept pair is the two largest keys,
// found with a min/max network.  The sign rides along in bit 0, below the
// index, where it cannot affect the order.  Returns the four codes (kept
// elements in ascending index order, group 0 first); `mb` receives the
// metadata byte, `dn` (DENSE) the 8 codes with zeros at pruned positions.
template <bool DENSE, class Code>
__device__ __forceinline__ uint32_t prune24_encode(const uint4 v, const Code &code, uint32_t &mb,
                                                   uint2 &dn) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
  mb = 0;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const uint32_t lo = w[2 * g], hi = w[2 * g + 1];
    // rotate the element's magnitude to bits 17..31 and its sign to bit 0
    const uint32_t k0 = (__funnelshift_l(lo, lo, 17) & 0xFFFE0001u) | (3u << 1);
    const uint32_t k1 = (__funnelshift_l(lo, lo, 1) & 0xFFFE0001u) | (2u << 1);
    const uint32_t k2 = (__funnelshift_l(hi, hi, 17) & 0xFFFE0001u) | (1u << 1);
    const uint32_t k3 = __funnelshift_l(hi, hi, 1) & 0xFFFE0001u;
    const uint32_t hi01 = max(k0, k1), lo01 = min(k0, k1);
    const uint32_t hi23 = max(k2, k3), lo23 = min(k2, k3);
    const uint32_t f = max(hi01, hi23);
    const uint32_t sc = max(min(hi01, hi23), max(lo01, lo23));
    // a = the kept element of lower index (larger 3 - i), b = the other one
    const bool f_lower = (f & 6u) > (sc & 6u);
    const uint32_t ka = f_lower ? f : sc, kb = f_lower ? sc : f;
    const uint32_t ia = 3u - ((ka >> 1) & 3u), ib = 3u - ((kb >> 1) & 3u);
    mb |= (ia | (ib << 2)) << (4 * g);
    const uint32_t ca = code((ka >> 17) | ((ka & 1u) << 15));
    const uint32_t cb = code((kb >> 17) | ((kb & 1u) << 15));
    out |= (ca | (cb << 8)) << (16 * g);
    if (DENSE) (g ? dn.y : dn.x) = (ca << (8 * ia)) | (cb << (8 * ib));
  }
  return out;
}

// The same selection with both groups in the two 16-bit lanes of a word,
// split over the two phases: phase 1 (memory-bound) selects and stores the
// metadata byte, phase 2 reads it back and only encodes the kept pair.
// A_i = (|w| of element i of group 1) << 16 | (|w| of element i of group 0);
// for j < i, (A_j | 0x80008000) - A_i has bit 15 (group 0) and bit 31
// (group 1) set exactly when |w_j| >= |w_i|, i.e. when j beats i (the lower
// index wins ties); when it is clear, i beats j.  The six such bits of a
// group decide the kept pair, so a 64-entry table maps them to the pair's
// metadata nibble.
__device__ __forceinline__ void build_select_tables(uint32_t *nib64, uint32_t *sel16, int t) {
  if (t < 64) {
    // bit order of the index: g01, g02, g03, g12, g13, g23 (g_ji = j beats i);
    // element i is kept when fewer than two elements beat it
    const int g01 = t & 1, g02 = (t >> 1) & 1, g03 = (t >> 2) & 1;
    const int g12 = (t >> 3) & 1, g13 = (t >> 4) & 1, g23 = (t >> 5) & 1;
    const int beaten0 = 3 - g01 - g02 - g03;
    const int beaten1 = g01 + 2 - g12 - g13;
    const int beaten2 = g02 + g12 + 1 - g23;
    const int beaten3 = g03 + g13 + g23;
    const uint32_t keep = (beaten0 < 2 ? 1u : 0u) | (beaten1 < 2 ? 2u : 0u) | (beaten2 < 2 ? 4u : 0u) |
                          (beaten3 < 2 ? 8u : 0u);
    uint32_t nib = 0;
    if (__popc(keep) == 2) {  // patterns that no input produces keep nibble 0
      const uint32_t lo = __ffs(keep) - 1, hi = 31 - __clz(keep);
      nib = lo | (hi << 2);
    }
    nib64[t] = nib * 17u;  // the nibble in both halves of the byte
  }
  // metadata nibble -> the byte-permute selector of its kept pair: element i
  // of a group is bytes 2i and 2i + 1 of the group's two words (16 words, one
  // per bank, so lookups never conflict)
  if (t < 16) {
    const uint32_t lo = t & 3u, hi = (t >> 2) & 3u;
    sel16[t] = (2 * lo) | ((2 * lo + 1) << 4) | ((2 * hi) << 8) | ((2 * hi + 1) << 12);
  }
}

// Phase 1: the metadata byte of a unit; amax2 accumulates the lane-wise
// largest magnitude bits (both halves of the word).
__device__ __forceinline__ uint32_t prune24_select(const uint4 v, const uint32_t *nib64, uint32_t &amax2) {
  const uint32_t a0 = __byte_perm(v.x, v.z, 0x5410), a1 = __byte_perm(v.x, v.z, 0x7632);
  const uint32_t a2 = __byte_perm(v.y, v.w, 0x5410), a3 = __byte_perm(v.y, v.w, 0x7632);
  constexpr uint32_t kMag = 0x7FFF7FFFu, kTop = 0x80008000u;
  const uint32_t m0 = a0 & kMag, m1 = a1 & kMag, m2 = a2 & kMag, m3 = a3 & kMag;
  amax2 = __vmaxu2(amax2, __vmaxu2(__vmaxu2(m0, m1), __vmaxu2(m2, m3)));
  const uint32_t h0 = a0 | kTop, h1 = a1 | kTop, h2 = a2 | kTop;
  uint32_t bits = (h0 - m1) & kTop;                        // g01
  bits = (bits >> 1) | ((h0 - m2) & kTop);                 // g02
  bits = (bits >> 1) | ((h0 - m3) & kTop);                 // g03
  bits = (bits >> 1) | ((h1 - m2) & kTop);                 // g12
  bits = (bits >> 1) | ((h1 - m3) & kTop);                 // g13
  bits = (bits >> 1) | ((h2 - m3) & kTop);                 // g23
  return (nib64[(bits >> 10) & 63u] & 0x0Fu) | (nib64[bits >> 26] & 0xF0u);
}

// Phase 2: the four E4M3 codes of a unit whose metadata byte is mb (kept
// elements in ascending index order, group 0 first).
template <class Code>
__device__ __forceinline__ uint32_t prune24_codes(const uint4 v, uint32_t mb, const uint32_t *sel16,
                                                  const Code &code) {
  const uint32_t p0 = __byte_perm(v.x, v.y, sel16[mb & 15u]);         // kept pair of group 0
  const uint32_t p1 = __byte_perm(v.z, v.w, sel16[(mb >> 4) & 15u]);  // and of group 1
  return code.codes4(p0, p1);
}

// Byte offset, in its packed block, of the 4 value bytes of unit u (row
// u / 16, columns 8 (u % 16) ..): row r's 16-byte chunk c sits at chunk
// position c ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t packed_value_offset(uint32_t u) {
  const uint32_t r = u >> 4, cchunk = (u >> 2) & 3u;
  return r * 64 + (((cchunk ^ (r >> 1)) & 3u) << 4) + (u & 3u) * 4;
}

// E4M3 2:4 ops whose selection runs in phase 1 (the DENSE variant selects and
// encodes in phase 2).
template <int OP, bool FP8, bool DENSE>
__host__ __device__ constexpr bool selects_in_phase1() {
  return OP == kOpPrune24Packed || (OP == kOpPrune24 && FP8 && !DENSE);
}

// Where phase 1 leaves a unit's 2:4 metadata byte for phase 2.
template <int OP>
__device__ __forceinline__ uint8_t *meta_byte(const StreamArgs &a, const Chunk &ch, uint32_t u) {
  if constexpr (OP == kOpPrune24Packed)
    return a.out + ch.idx * kPackedBlockBytes + 128 * 64 + u;
  else
    return a.meta + (ch.e >> 3) + u;
}

// kOpSlide68Packed: where unit u of chunk `ch` lands.  Row r of row tile t,
// K'-group kg (three packed blocks); the unit is 16 W columns = 24 K'
// columns: value bytes 12 j .. 12 j + 11 and metadata bytes 3 j .. 3 j + 2 of
// the group's 192 / 48 bytes per row (j = unit in the row).
struct Slide68Place {
  uint8_t *group;  // packed block (t, 3 kg)
  uint32_t r, j;
};

// the chunk's packed block group and first row, once per chunk:
// chunk c = (t K/256 + kg) 2 + h covers rows 64 h .. of row tile t
__device__ __forceinline__ void slide68_chunk(const StreamArgs &a, Chunk &ch) {
  const uint32_t kgroups = a.kblocks / 3;
  const uint32_t c = static_cast<uint32_t>(ch.idx);
  const uint32_t t = c / (2 * kgroups), rem = c - t * (2 * kgroups);
  ch.group = a.out + (static_cast<uint64_t>(t) * a.kblocks + 3 * (rem >> 1)) * kPackedBlockBytes;
  ch.row0 = 64 * (rem & 1u);
}

__device__ __forceinline__ Slide68Place slide68_place(const StreamArgs &, const Chunk &ch, uint32_t u) {
  return Slide68Place{ch.group, ch.row0 + (u >> 4), u & 15u};
}

// metadata byte b (0..47) of the place's row
__device__ __forceinline__ uint8_t *slide68_meta_at(const Slide68Place &pl, uint32_t b) {
  return pl.group + (b >> 4) * kPackedBlockBytes + 128 * 64 + pl.r * 16 + (b & 15u);
}

// 4-byte value word at row byte o (0..188, a multiple of 4) of the place's row,
// inside the 64-byte-swizzled chunk placement of its block
__device__ __forceinline__ uint32_t *slide68_value_at(const Slide68Place &pl, uint32_t o) {
  const uint32_t ob = o & 63u;
  return reinterpret_cast<uint32_t *>(pl.group + (o >> 6) * kPackedBlockBytes + pl.r * 64 +
                                      ((((ob >> 4) ^ (pl.r >> 1)) & 3u) << 4) + (ob & 15u));
}

// ------------------------------------------------------------------ phase 1
// One unit: `p` its bytes in shared memory, u its index in chunk `ch`; mx2
// accumulates the per-lane largest magnitude bits.
template <int OP, bool FP8, bool DENSE>
__device__ __forceinline__ void phase1_unit(const uint8_t *p, const Chunk &ch, uint32_t u,
                                            const StreamArgs &a, const uint32_t *nib64, uint32_t &mx2) {
  if constexpr (OP == kOpSlide68 || OP == kOpSlide68Packed) {
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
    if constexpr (OP == kOpSlide68Packed) {
      const Slide68Place pl = slide68_place(a, ch, u);
#pragma unroll
      for (int b = 0; b < 3; ++b)
        *slide68_meta_at(pl, 3 * pl.j + b) = static_cast<uint8_t>(nib[2 * b] | (nib[2 * b + 1] << 4));
    } else {
      uint8_t *m = a.meta + 3 * (ch.e >> 4) + 3 * u;
      m[0] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
      m[1] = static_cast<uint8_t>(nib[2] | (nib[3] << 4));
      m[2] = static_cast<uint8_t>(nib[4] | (nib[5] << 4));
    }
    if (!FP8) {
      uint2 *d = reinterpret_cast<uint2 *>(a.out + 24 * (ch.e >> 4) + 24 * u);
#pragma unroll
      for (int o = 0; o < 3; ++o)
        d[o] = make_uint2(vals[4 * o] | (vals[4 * o + 1] << 16), vals[4 * o + 2] | (vals[4 * o + 3] << 16));
    }
    mx2 = __vmaxu2(mx2, __vmaxu2(absmax8x2(v0), absmax8x2(v1)));
  } else {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    if constexpr (selects_in_phase1<OP, FP8, DENSE>()) {
      *meta_byte<OP>(a, ch, u) = static_cast<uint8_t>(prune24_select(v, nib64, mx2));
      return;
    } else if constexpr (OP == kOpPrune24 && !FP8) {
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
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (t == i0) kept[2 * g] = h[4 * g + t];
          if (t == i1) kept[2 * g + 1] = h[4 * g + t];
          if (DENSE) dn[4 * g + t] = ((mk >> t) & 1u) ? h[4 * g + t] : 0u;
        }
      }
      a.meta[(ch.e >> 3) + u] = static_cast<uint8_t>(mb);
      *reinterpret_cast<uint2 *>(a.out + ch.e + 8 * u) =
          make_uint2(kept[0] | (kept[1] << 16), kept[2] | (kept[3] << 16));
      if (DENSE)
        *reinterpret_cast<uint4 *>(a.dense + 2 * ch.e + 16 * u) =
            make_uint4(dn[0] | (dn[1] << 16), dn[2] | (dn[3] << 16), dn[4] | (dn[5] << 16),
                       dn[6] | (dn[7] << 16));
    }
    mx2 = __vmaxu2(mx2, absmax8x2(v));
  }
}

// ------------------------------------------------------------------ phase 2
// `meta_in` is the unit's metadata (one byte for 2:4, three for 6:8), loaded
// before the chunk's stores so that the loads overlap.
template <int OP, bool DENSE, class Code>
__device__ __forceinline__ void phase2_unit(const uint8_t *p, const Chunk &ch, uint32_t u, uint32_t meta_in,
                                            const StreamArgs &a, const Code &code, const uint32_t *sel16) {
  if constexpr (OP == kOpSlide68 || OP == kOpSlide68Packed) {
    const uint4 v0 = reinterpret_cast<const uint4 *>(p)[0];
    const uint4 v1 = reinterpret_cast<const uint4 *>(p)[1];
    const uint32_t m3 = meta_in;
    // wp[3 gl + j] = the two kept values of window j of 8-group gl (low half
    // first): the unit's 12 codes in output order, encoded four at a time
    uint32_t wp[6];
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
        wp[3 * gl + j] = h0 | (h1 << 16);
      }
    }
    uint32_t c[3];
#pragma unroll
    for (int o = 0; o < 3; ++o) c[o] = code.codes4(wp[2 * o], wp[2 * o + 1]);
    if constexpr (OP == kOpSlide68Packed) {
      const Slide68Place pl = slide68_place(a, ch, u);
#pragma unroll
      for (int o = 0; o < 3; ++o) *slide68_value_at(pl, 12 * pl.j + 4 * o) = c[o];
    } else {
      uint32_t *d = reinterpret_cast<uint32_t *>(a.out + 12 * (ch.e >> 4) + 12 * u);
#pragma unroll
      for (int o = 0; o < 3; ++o) d[o] = c[o];
    }
  } else {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    if constexpr (OP == kOpPrune24Packed) {
      *reinterpret_cast<uint32_t *>(a.out + ch.idx * kPackedBlockBytes + packed_value_offset(u)) =
          prune24_codes(v, meta_in, sel16, code);
    } else if constexpr (OP == kOpPrune24 && !DENSE) {
      *reinterpret_cast<uint32_t *>(a.out + (ch.e >> 1) + 4 * u) = prune24_codes(v, meta_in, sel16, code);
    } else if constexpr (OP == kOpPrune24) {
      uint32_t mb;
      uint2 dn;
      *reinterpret_cast<uint32_t *>(a.out + (ch.e >> 1) + 4 * u) = prune24_encode<true>(v, code, mb, dn);
      *reinterpret_cast<uint2 *>(a.dense + ch.e + 8 * u) = dn;
      a.meta[(ch.e >> 3) + u] = static_cast<uint8_t>(mb);
    } else {
      const uint32_t c03 = code.codes4(v.x, v.y), c47 = code.codes4(v.z, v.w);
      if constexpr (OP == kOpQuantize) {
        *reinterpret_cast<uint2 *>(a.out + ch.e + 8 * u) = make_uint2(c03, c47);
      } else if constexpr (OP == kOpLift) {
        // lifted[12 g + 4 j + r] = code(x[8 g + 2 j + r]) for the 8-group g
        uint32_t *d = reinterpret_cast<uint32_t *>(a.out + 12 * (ch.e >> 3) + 12 * u);
        d[0] = c03;
        d[1] = __byte_perm(c03, c47, 0x5432);  // codes 2..5
        d[2] = c47;
      }
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int OP, bool FP8, bool DENSE, bool SMALL>
__global__ void __launch_bounds__(kThreads, 1) stream_kernel(const __grid_constant__ StreamArgs a) {
  constexpr int kS = ring_stages<SMALL>();
  constexpr int kUnit = unit_bytes<OP>();
  constexpr int kRows = kChunkBytes / (kConsumers * kUnit);  // units per thread per chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  uint8_t *tab = ring + kS * kChunkBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(tab + table_bytes<SMALL>());
  uint64_t *empty = full + kS;
  __shared__ uint32_t s_red[kConsumers / 32];
  __shared__ uint32_t s_nib64[64];    // 2:4: comparison bits -> metadata nibble
  __shared__ uint32_t s_sel16[16];    // 2:4: metadata nibble -> byte-permute selector
  __shared__ uint32_t s_amax;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * a.nchunks / gridDim.x;
  const int64_t c1 = static_cast<int64_t>(blockIdx.x + 1) * a.nchunks / gridDim.x;
  const int n_my = static_cast<int>(c1 - c0);
  const bool resident = n_my <= kS;                  // phase 2 reuses the ring contents
  const int n_loads = (FP8 && !resident) ? 2 * n_my : n_my;

  if (tid == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    fence_mbar_init();
  }
  if constexpr (selects_in_phase1<OP, FP8, DENSE>()) build_select_tables(s_nib64, s_sel16, tid);
  __syncthreads();
  grid_dependency_wait();
  // Activation kernels let the next kernel (a GEMM) launch early; the weight
  // path never does, which is what allows a GEMM to prefetch weights before
  // its own dependency wait.
  if (OP == kOpQuantize || OP == kOpLift) grid_launch_dependents();

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    // Load L < n_my brings chunk c0 + L, load n_my + i chunk c0 + n_my - 1 - i
    // (phase 2 walks the range backwards), into slot L % kS.  The second
    // pass is prefetched as soon as slots free up.
    if ((tid & 31) == 0) {
      if constexpr (OP == kOpPrune24Packed || OP == kOpSlide68Packed) prefetch_tensormap(&a.wmap);
      for (int L = 0; L < n_loads; ++L) {
        const int slot = L % kS;
        if (L >= kS && !mbar_wait(&empty[slot], static_cast<uint32_t>(L / kS - 1) & 1u, a.status))
          break;
        const int64_t c = L < n_my ? c0 + L : c0 + 2 * n_my - 1 - L;
        const uint32_t nb =
            static_cast<uint32_t>(min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes));
        mbar_arrive_expect_tx(&full[slot], nb);
        if constexpr (OP == kOpPrune24Packed) {
          const uint32_t t = static_cast<uint32_t>(c) / a.kblocks;
          const uint32_t kb = static_cast<uint32_t>(c) - t * a.kblocks;
          tma_load_2d(ring + slot * kChunkBytes, &a.wmap, &full[slot], static_cast<int32_t>(kb * 128),
                      static_cast<int32_t>(t * 128), l2_policy_evict_normal());
        } else if constexpr (OP == kOpSlide68Packed) {
          const uint32_t kgroups = a.kblocks / 3;
          const uint32_t t = static_cast<uint32_t>(c) / (2 * kgroups);
          const uint32_t rem = static_cast<uint32_t>(c) - t * (2 * kgroups);
          tma_load_2d(ring + slot * kChunkBytes, &a.wmap, &full[slot], static_cast<int32_t>((rem >> 1) * 256),
                      static_cast<int32_t>(t * 128 + (rem & 1u) * 64), l2_policy_evict_normal());
        } else {
          bulk_load(ring + slot * kChunkBytes, a.x + c * kChunkBytes, nb, &full[slot]);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // fn(unit bytes in shared memory, unit index) for this thread's units of
  // chunk c; full chunks (all but possibly the tensor's last) need no checks.
  auto for_units = [&](const uint8_t *chunk, int64_t c, auto &&fn) {
    const int64_t nb = min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes);
    if (nb == kChunkBytes) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const uint32_t u = static_cast<uint32_t>(r * kConsumers + tid);
        fn(chunk + u * kUnit, u);
      }
    } else {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const uint32_t u = static_cast<uint32_t>(r * kConsumers + tid);
        if (static_cast<int64_t>(u) * kUnit < nb) fn(chunk + u * kUnit, u);
      }
    }
  };
  auto chunk_of = [&](int64_t c) {
    Chunk ch{static_cast<uint64_t>(c) * (kChunkBytes / 2), static_cast<uint64_t>(c), nullptr, 0};
    if constexpr (OP == kOpSlide68Packed) slide68_chunk(a, ch);
    return ch;
  };

  // The table costs about as much as dividing 2 chunks' elements directly.
  constexpr bool kQuot = quot_encoder<OP, DENSE>();
  const bool direct = SMALL || n_my <= 2;
  if constexpr (FP8 && !SMALL && !kQuot) {
    if (!direct) zero_table(tab, tid);  // ordered before its entries by the barriers below
  }

  uint32_t mx2 = 0;  // per-lane largest magnitude bits
  for (int i = 0; i < n_my; ++i) {
    const int slot = i % kS;
    mbar_wait(&full[slot], static_cast<uint32_t>(i / kS) & 1u, a.status);
    const Chunk ch = chunk_of(c0 + i);
    for_units(ring + slot * kChunkBytes, c0 + i, [&](const uint8_t *p, uint32_t u) {
      phase1_unit<OP, FP8, DENSE>(p, ch, u, a, s_nib64, mx2);
    });
    __syncwarp();
    if (!resident && (tid & 31) == 0) mbar_arrive(&empty[slot]);
  }
  uint32_t mx = max(mx2 & 0xFFFFu, mx2 >> 16);
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
    // The amax and the arrival are posted without waiting (the release on the
    // arrival orders the max before it); the departure count that lets the
    // last CTA re-zero the counters is taken at the end of the kernel, off
    // the critical path.
    if (tid == 0) {
      red_max_relaxed_gpu(&a.ws[0], mx);
      red_add_release_gpu(&a.ws[1], 1u);
      const uint64_t t0 = global_timer_ns();
      uint32_t polls = 0;
      while (ld_acquire_u32(&a.ws[1]) < gridDim.x) {
        __nanosleep(32);
        if ((++polls & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
          if (a.status) atomicOr(a.status, SP24_STATUS_TIMEOUT);
          break;
        }
      }
      const uint32_t amax = ld_acquire_u32(&a.ws[0]);
      s_amax = amax;
      if (blockIdx.x == 0) {
        if (amax >= 0x7F80u && a.status) atomicOr(a.status, SP24_STATUS_NONFINITE);
        if (a.scale_out) *a.scale_out = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
      }
    }
    named_bar_sync(1, kConsumers);
    const uint32_t amax = s_amax;
    const float s = amax == 0u ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax), 448.0f);
    if constexpr (!SMALL && !kQuot) {
      if (!direct) fill_table(tab, amax, s, tid);
    }
    named_bar_sync(1, kConsumers);

    // ---------------------------------------------------------- phase 2
    // The units' metadata (1 byte for 2:4, 3 for 6:8; this thread wrote it in
    // phase 1) of chunk c, loaded one chunk ahead so the L2 latency overlaps
    // the previous chunk's work.
    constexpr bool kMetaIn = OP == kOpSlide68 || OP == kOpSlide68Packed || selects_in_phase1<OP, FP8, DENSE>();
    auto load_meta = [&](int64_t c, uint32_t (&m)[kRows]) {
      const Chunk ch = chunk_of(c);
      const int64_t nb = min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const uint32_t u = static_cast<uint32_t>(r * kConsumers + tid);
        m[r] = 0;
        if (static_cast<int64_t>(u) * kUnit < nb) {
          if constexpr (OP == kOpSlide68) {
            const uint8_t *mp = a.meta + 3 * (ch.e >> 4) + 3 * u;
            m[r] = __ldcg(mp) | (static_cast<uint32_t>(__ldcg(mp + 1)) << 8) |
                   (static_cast<uint32_t>(__ldcg(mp + 2)) << 16);
          } else if constexpr (OP == kOpSlide68Packed) {
            const Slide68Place pl = slide68_place(a, ch, u);
            m[r] = __ldcg(slide68_meta_at(pl, 3 * pl.j)) |
                   (static_cast<uint32_t>(__ldcg(slide68_meta_at(pl, 3 * pl.j + 1))) << 8) |
                   (static_cast<uint32_t>(__ldcg(slide68_meta_at(pl, 3 * pl.j + 2))) << 16);
          } else {
            m[r] = __ldcg(meta_byte<OP>(a, ch, u));
          }
        }
      }
    };

    // ---------------------------------------------------------- phase 2
    auto phase2 = [&](const auto &code) {
      [[maybe_unused]] uint32_t mnext[kRows];
      if constexpr (kMetaIn) load_meta(c0 + n_my - 1, mnext);
      for (int i = 0; i < n_my; ++i) {
        const int j = n_my - 1 - i;  // chunk of the range, last first
        int slot = j;                // resident: where phase 1 left it
        const int L = n_my + i;
        [[maybe_unused]] uint32_t mrow[kRows];
        if constexpr (kMetaIn) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) mrow[r] = mnext[r];
          if (j > 0) load_meta(c0 + j - 1, mnext);
        }
        if (!resident) {
          slot = L % kS;
          mbar_wait(&full[slot], static_cast<uint32_t>(L / kS) & 1u, a.status);
        }
        const int64_t c = c0 + j;
        const Chunk ch = chunk_of(c);
        const uint8_t *chunk = ring + slot * kChunkBytes;
        if constexpr (kMetaIn) {
          const int64_t nb = min(static_cast<int64_t>(kChunkBytes), a.nbytes - c * kChunkBytes);
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const uint32_t u = static_cast<uint32_t>(r * kConsumers + tid);
            if (static_cast<int64_t>(u) * kUnit < nb)
              phase2_unit<OP, DENSE>(chunk + u * kUnit, ch, u, mrow[r], a, code, s_sel16);
          }
        } else {
          for_units(chunk, c, [&](const uint8_t *p, uint32_t u) {
            phase2_unit<OP, DENSE>(p, ch, u, 0u, a, code, s_sel16);
          });
        }
        __syncwarp();
        if (!resident && (tid & 31) == 0) mbar_arrive(&empty[slot]);
      }
    };
    if constexpr (kQuot) {
      phase2(CodeQuot{s, __frcp_rn(s)});
    } else if constexpr (SMALL) {
      phase2(CodeTable<true>{tab, s});
    } else {
      if (direct)
        phase2(CodeTable<true>{tab, s});
      else
        phase2(CodeTable<false>{tab, s});
    }
    if (tid == 0) {
      __threadfence();
      if (atomicAdd(&a.ws[2], 1u) == gridDim.x - 1) {  // last to leave: re-zero the counters
        a.ws[0] = 0u;
        a.ws[1] = 0u;
        a.ws[2] = 0u;
      }
    }
  }
}

template <int OP, bool FP8, bool DENSE, bool SMALL>
cudaError_t launch_stream_variant(const StreamArgs &a, int64_t grid, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(stream_kernel<OP, FP8, DENSE, SMALL>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<SMALL>());
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<SMALL>();
  cfg.stream = st;
  // Cooperative: only the two-phase kernels wait on each other.
  // Programmatic dependent launch: the grid may start while the previous
  // kernel finishes; every CTA passes griddepcontrol.wait before touching
  // memory.
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (FP8) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, stream_kernel<OP, FP8, DENSE, SMALL>, a);
}

template <int OP, bool FP8, bool DENSE>
cudaError_t launch_stream_typed(const StreamArgs &a, int sm_count, cudaStream_t st) {
  int64_t grid = a.nchunks < sm_count ? a.nchunks : sm_count;
  if (grid < 1) grid = 1;
  const int64_t per_cta = (a.nchunks + grid - 1) / grid;
  return per_cta <= 2 ? launch_stream_variant<OP, FP8, DENSE, true>(a, grid, st)
                      : launch_stream_variant<OP, FP8, DENSE, false>(a, grid, st);
}

StreamArgs make_args(const void *x, int64_t nelem, uint32_t *ws, float *scale, int32_t *status,
                     void *out, uint8_t *meta, void *dense) {
  StreamArgs a;
  memset(&a, 0, sizeof(a));
  a.x = static_cast<const uint8_t *>(x);
  a.nbytes = nelem * 2;
  a.nchunks = (a.nbytes + kChunkBytes - 1) / kChunkBytes;
  a.ws = ws;
  a.scale_out = scale;
  a.status = status;
  a.out = static_cast<uint8_t *>(out);
  a.meta = meta;
  a.dense = static_cast<uint8_t *>(dense);
  a.kblocks = 0;
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

cudaError_t launch_prune24_packed_fused(const void *w, int N, int K, uint32_t *ws, float *scale,
                                        uint8_t *packed, int32_t *status, int sm_count,
                                        cudaStream_t st) {
  StreamArgs a = make_args(w, static_cast<int64_t>(N) * K, ws, scale, status, packed, nullptr, nullptr);
  a.kblocks = static_cast<uint32_t>(K / 128);
  // chunk = one 128-row x 128-column box of W = the input of one packed block
  static_assert(kChunkBytes == 128 * 128 * 2, "a chunk must be one packed block's input");
  if (!make_tensor_map_2d(&a.wmap, w, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, static_cast<uint64_t>(K),
                          static_cast<uint64_t>(N), 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  return launch_stream_typed<kOpPrune24Packed, true, false>(a, sm_count, st);
}

cudaError_t launch_slide68_packed_fused(const void *w, int N, int K, uint32_t *ws, float *scale,
                                        uint8_t *packed, int32_t *status, int sm_count,
                                        cudaStream_t st) {
  StreamArgs a = make_args(w, static_cast<int64_t>(N) * K, ws, scale, status, packed, nullptr, nullptr);
  a.kblocks = static_cast<uint32_t>(3 * K / 256);  // K' / 128
  // chunk = 64 rows x 256 columns of W = rows 64 h .. of three packed blocks
  static_assert(kChunkBytes == 64 * 256 * 2, "a chunk must be half the input of three packed blocks");
  if (!make_tensor_map_2d(&a.wmap, w, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, static_cast<uint64_t>(K),
                          static_cast<uint64_t>(N), 256, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  return launch_stream_typed<kOpSlide68Packed, true, false>(a, sm_count, st);
}

cudaError_t launch_slide68_fused(const void *w, int64_t nelem, bool fp8, uint32_t *ws,
                                 float *scale, void *values, uint8_t *meta, int32_t *status,
                                 int sm_count, cudaStream_t st) {
  const StreamArgs a = make_args(w, nelem, ws, scale, status, values, meta, nullptr);
  return fp8 ? launch_stream_typed<kOpSlide68, true, false>(a, sm_count, st)
             : launch_stream_typed<kOpSlide68, false, false>(a, sm_count, st);
}

}  // namespace sp24
