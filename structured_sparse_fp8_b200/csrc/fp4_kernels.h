// fp4_kernels.h -- launchers of the FP4 (E2M1) kernels (fp4.cu).  `ws` is
// at least two zero 32-bit words of workspace (amax, departures), zero again
// when the launches complete.  Codes are packed two per byte, element 2i in
// the low nibble of byte i.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sp24 {

// X bf16 [nelem] (nelem % 8 == 0) -> q [nelem / 2] bytes, scale <- amax / 6.
cudaError_t launch_fp4_quantize(const void *x, int64_t nelem, uint32_t *ws, float *scale, uint8_t *q,
                                int32_t *status, int sms, cudaStream_t st);

// W bf16 [N, K] (nelem = N K, K % 8 == 0) -> 2:4 values [N, K/2] codes
// ([N, K/4] bytes) and metadata [N, K/8] in the canonical layout,
// scale <- amax / 6.
cudaError_t launch_fp4_prune24(const void *w, int64_t nelem, uint32_t *ws, float *scale, uint8_t *values,
                               uint8_t *meta, int32_t *status, int sms, cudaStream_t st);

}  // namespace sp24
