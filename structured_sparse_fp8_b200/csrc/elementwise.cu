// elementwise.cu -- small helper kernels outside the streamed path:
//   * the E4M3 encoder applied to fp32 values (a test hook that pins the
//     device rounding against the oracle),
//   * the re-layout of canonical 2:4 E4M3 weights into the GEMM's
//     tile-packed blocks.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "quant_common.cuh"

namespace sp24 {

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
