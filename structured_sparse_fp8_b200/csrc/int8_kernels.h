// int8_kernels.h -- launchers of the INT8 W8A8 kernels (int8.cu).  `ws` is
// at least two zero 32-bit words of workspace (amax, departures), zero again
// when the launches complete.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sp24 {

// X bf16 [nelem] (nelem % 8 == 0) -> q int8 [nelem], scale <- amax / 127.
cudaError_t launch_int8_quantize(const void *x, int64_t nelem, uint32_t *ws, float *scale, int8_t *q,
                                 int32_t *status, int sms, cudaStream_t st);

// W bf16 [N, K] (nelem = N K, K % 8 == 0) -> 2:4 values int8 [N, K/2] and
// metadata [N, K/8] in the canonical layout, scale <- amax / 127.
cudaError_t launch_int8_prune24(const void *w, int64_t nelem, uint32_t *ws, float *scale, int8_t *values,
                                uint8_t *meta, int32_t *status, int sms, cudaStream_t st);

}  // namespace sp24
