// noalloc.cu -- per-tensor E4M3 quantisation for callers that cannot allocate
// device memory.
//
// fp8_quantize_pertensor needs a small zero-initialised scratch area for its
// amax reduction (a running maximum and a finished-block counter), which the
// caller normally passes as `workspace`.  Some callers cannot provide one: an
// engine or plugin host that owns every device allocation and forbids its
// plugins from calling cudaMalloc, or a latency-critical loop where the
// implicit device synchronisation of cudaMalloc/cudaFree is not acceptable.
// This file gives them fp8_quantize_pertensor_static: a decode-sized X goes
// to the one-cluster quantiser, which needs no scratch at all; a larger X
// keeps its scratch in a file-scope __device__ array instead.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "sp24.h"

namespace sp24 {
// SM count of the current device, or -1 when it is not sm_100 (api.cu; looked
// up once per device).
int current_device_sm_count();
}  // namespace sp24

namespace {

// Scratch of the static-scratch entry point.  Every GPU that loads the
// library holds these bytes until the process exits.
constexpr size_t kStaticScratchBytes = 256;
static_assert(sp24::kAmaxWorkspaceBytes <= kStaticScratchBytes, "static scratch too small");
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

}  // namespace

extern "C" int fp8_quantize_pertensor_static(const void *X, int64_t rows, int64_t cols,
                                             uint8_t *q, float *scale, int32_t *status,
                                             sp24_stream_t stream) {
  if (!X || !q || !scale) return SP24_ERR_NULL;
  if (rows < 1 || cols < 1 || cols % 16 != 0) return SP24_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(X) & 15u) || (reinterpret_cast<uintptr_t>(q) & 15u))
    return SP24_ERR_ALIGN;
  // The scratch this call needs does not grow with the tensor; reject any
  // configuration whose need would exceed the static array.
  if (sp24_workspace_size(SP24_OP_QUANTIZE, rows, 0, cols, SP24_DTYPE_E4M3) > kStaticScratchBytes)
    return SP24_ERR_WORKSPACE;
  const int sms = sp24::current_device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nelem = rows * cols;
  cudaError_t e;
  if (sp24::small_quantize_fits(nelem)) {
    e = sp24::launch_quantize_small(X, nelem, sp24::kSmallE4M3, scale, q, status, st);
  } else {
    // In host code `g_static_scratch` names a host-side stand-in; the device
    // address is looked up on every call (cheap once the module is loaded),
    // so that a context created after a reset never gets a stale one.
    void *scratch = nullptr;
    e = cudaGetSymbolAddress(&scratch, g_static_scratch);
    // The array keeps whatever the previous call left (a timed-out call's
    // counters): clear them.  This copy sits on the stream between the
    // previous kernel and the quantiser, which therefore cannot start early
    // beside that kernel (programmatic launch) as it does with a workspace.
    if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, sp24::kAmaxWorkspaceBytes, st);
    if (e == cudaSuccess)
      e = sp24::launch_quantize_fused(X, nelem, static_cast<uint32_t *>(scratch), scale, q, status, sms, st);
  }
  if (e != cudaSuccess) {
    sp24::set_last_cuda_error(static_cast<int>(e));
    return SP24_ERR_CUDA;
  }
  return SP24_OK;
}
