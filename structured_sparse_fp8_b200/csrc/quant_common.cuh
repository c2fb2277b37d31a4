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
