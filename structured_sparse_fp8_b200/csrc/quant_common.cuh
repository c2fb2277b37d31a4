// quant_common.cuh -- device helpers shared by the elementwise kernels:
// streaming loads, bf16 -> fp32, the E4M3 encoder, and the magnitude
// selections of 2:4 and 6:8 pruning.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sp24 {

// ----------------------------------------------------------------- helpers

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// E4M3 code of one fp32 value: round to nearest even, saturate to +-448, and
// keep the sign of a value that rounds to zero (code 0x80 for negatives).
// A NaN of either sign gives 0x7F: finite values saturate at magnitude code
// 0x7E, so a magnitude code of 0x7F is the conversion's NaN, whatever sign it
// carries, and it is returned without one.
__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  const uint32_t c = r & 0xFFu;
  return (c & 0x7Fu) == 0x7Fu ? 0x7Fu : c | ((__float_as_uint(v) >> 24) & 0x80u);
}

// E4M3 codes of RN_fp32(x / s) without a division on the common path.
// r = RN(1 / s) is given.  q = RN(x * r) differs from x / s by less than
// three units of x / s's last place (two roundings of relative size 2^-24
// each), so at most six fp32 steps from RN(x / s) even across a binade
// edge.  E4M3 rounding is monotone in the value, so when the fp32 values
// eight steps either side of q have the same code, RN(x / s) has it too.
// The check runs on four codes at once (one byte each); when it fails for
// any of them (a rounding boundary within reach, about one value in 2^16;
// NaN or Inf) the correctly rounded division decides all four.  The result
// is exactly e4m3_code(__fdiv_rn(x, s)) for every x and s > 0.

// The E4M3 codes of fp32 values hi and lo, in bits 8-15 and 0-7.
__device__ __forceinline__ uint32_t e4m3_pair(float hi, float lo) {
  uint16_t pr;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(hi), "f"(lo));
  return pr;
}

// Codes of the four bf16 values of h0 (elements 0, 1) and h1 (2, 3), byte i
// = element i; false when the division must decide.
__device__ __forceinline__ bool e4m3_codes4_quot(uint32_t h0, uint32_t h1, float r, uint32_t &out) {
  const uint32_t hh[4] = {h0 & 0xFFFFu, h0 >> 16, h1 & 0xFFFFu, h1 >> 16};
  uint32_t p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u = __float_as_uint(__fmul_rn(bf16_bits_to_float(hh[i]), r));
    const uint32_t mag = u & 0x7FFFFFFFu, sgn = u & 0x80000000u;
    p[i] = e4m3_pair(__uint_as_float(sgn | (mag + 8u)), __uint_as_float(sgn | (mag > 8u ? mag - 8u : 0u)));
  }
  // bytes (low, high) of each pair: the codes 8 steps below and above q
  const uint32_t w01 = p[0] | p[1] << 16, w23 = p[2] | p[3] << 16;
  const uint32_t lo = __byte_perm(w01, w23, 0x6420), hi = __byte_perm(w01, w23, 0x7531);
  // both ends equal, and no NaN code (magnitude 0x7F)
  const uint32_t bad = (lo ^ hi) | (((lo & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u);
  // the sign of every input (a value that rounds to zero keeps it)
  out = lo | (__byte_perm(h0, h1, 0x7531) & 0x80808080u);
  return bad == 0u;
}

// INT8 code of the bf16 pattern h at scale s: the correctly rounded quotient
// rounded half to even and clamped to +-127.
__device__ __forceinline__ int32_t int8_code(uint32_t h, float s) {
  const int32_t q = __float2int_rn(__fdiv_rn(bf16_bits_to_float(h), s));
  return min(max(q, -127), 127);
}

// E2M1 code (4 bits) of one fp32 value.  Both halves of the pair convert the
// same value, so the result does not depend on which half lands in which
// nibble; the sign is ORed in for a value that rounds to zero.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\tcvt.u16.u8 %0, t;\n\t}" : "=h"(r) : "f"(v));
  return (r & 0x7u) | ((__float_as_uint(v) >> 28) & 0x8u);
}

// The exact forms, out of line: rare, and kept out of the unrolled loops.
static __device__ __noinline__ uint32_t e4m3_codes4_div(uint32_t h0, uint32_t h1, float s) {
  const uint32_t hh[4] = {h0 & 0xFFFFu, h0 >> 16, h1 & 0xFFFFu, h1 >> 16};
  uint32_t q = 0u;
  for (int i = 0; i < 4; ++i) q |= e4m3_code(__fdiv_rn(bf16_bits_to_float(hh[i]), s)) << (8 * i);
  return q;
}

static __device__ __noinline__ uint2 e4m3_codes8_div(const uint4 w, float s) {
  const uint32_t h[4] = {w.x, w.y, w.z, w.w};
  uint32_t q[2] = {0u, 0u};
  for (int i = 0; i < 8; ++i)
    q[i >> 2] |= e4m3_code(__fdiv_rn(bf16_bits_to_float((h[i >> 1] >> (16 * (i & 1))) & 0xFFFFu), s)) << (8 * (i & 3));
  return make_uint2(q[0], q[1]);
}

// The codes of the 8 bf16 values of a 16-byte vector, packed little-endian
// into two words, by the fast path; `ok` is false when e4m3_codes8_div must
// produce them instead.  No call and no branch: a caller encoding several
// vectors runs their fast paths interleaved and redoes the (rare) failed
// vectors afterwards.
__device__ __forceinline__ uint2 e4m3_codes8_fast(const uint4 w, float r, bool &ok) {
  uint32_t a, b;
  const bool oa = e4m3_codes4_quot(w.x, w.y, r, a);
  const bool ob = e4m3_codes4_quot(w.z, w.w, r, b);
  ok = oa && ob;
  return make_uint2(a, b);
}

// Largest magnitude bit patterns of the 8 bf16 values of a 16-byte vector,
// per 16-bit lane (the larger lane is the vector's).  For finite bf16 the
// unsigned order of (bits & 0x7FFF) is the order of |x|; NaN/Inf patterns
// (>= 0x7F80) sort above every finite value.
__device__ __forceinline__ uint32_t absmax8x2(uint4 v) {
  const uint32_t m = 0x7FFF7FFFu;
  return __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
}

// Kept-position mask (4 bits) of one group: element i is kept when fewer than
// two elements beat it (larger |w|, or equal |w| at a lower index).  With the
// unique keys k_i = |w_i| << 2 | (3 - i) "beats" is plain ">", so the kept pair
// is the two largest keys, found with a min/max network.
__device__ __forceinline__ uint32_t keep2of4(const uint32_t a[4]) {
  const uint32_t k0 = (a[0] << 2) | 3u, k1 = (a[1] << 2) | 2u;
  const uint32_t k2 = (a[2] << 2) | 1u, k3 = a[3] << 2;
  const uint32_t hi01 = max(k0, k1), lo01 = min(k0, k1);
  const uint32_t hi23 = max(k2, k3), lo23 = min(k2, k3);
  const uint32_t first = max(hi01, hi23);
  const uint32_t second = max(min(hi01, hi23), max(lo01, lo23));
  return (1u << (3u - (first & 3u))) | (1u << (3u - (second & 3u)));
}

// 6:8 keep mask (8 bits): element i is kept when fewer than six elements beat
// it, i.e. everything but the two smallest unique keys k_i = |w_i| << 3 | (7 - i).
__device__ __forceinline__ uint32_t keep6of8(const uint32_t a[8]) {
  uint32_t k[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) k[i] = (a[i] << 3) | static_cast<uint32_t>(7 - i);
  uint32_t lo1 = min(min(min(k[0], k[1]), min(k[2], k[3])), min(min(k[4], k[5]), min(k[6], k[7])));
  uint32_t lo2 = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < 8; ++i) lo2 = min(lo2, k[i] == lo1 ? 0xFFFFFFFFu : k[i]);
  return 0xFFu & ~((1u << (7u - (lo1 & 7u))) | (1u << (7u - (lo2 & 7u))));
}

// Greedy window assignment: window j (positions 2j..2j+3) takes the two
// lowest kept positions in its range that no earlier window took.
// pos[2j], pos[2j+1] receive the positions, ascending.
__device__ __forceinline__ void assign_windows(uint32_t kept, int pos[6]) {
  uint32_t left = kept;
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    uint32_t cand = left & (0xFu << (2 * j));
    const int p0 = __ffs(cand) - 1;
    cand &= cand - 1;
    const int p1 = __ffs(cand) - 1;
    pos[2 * j] = p0;
    pos[2 * j + 1] = p1;
    left &= ~((1u << p0) | (1u << p1));
  }
}

}  // namespace sp24
