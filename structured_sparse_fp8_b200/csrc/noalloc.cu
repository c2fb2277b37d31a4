// noalloc.cu -- per-tensor E4M3 quantisation for callers that cannot allocate
// device memory.
//
// fp8_quantize_pertensor needs a small zero-initialised scratch area for its
// amax reduction (a running maximum and a finished-block counter), which the
// caller normally passes as `workspace`.  Some callers cannot provide one: an
// engine or plugin host that owns every device allocation and forbids its
// plugins from calling cudaMalloc, or a latency-critical loop where the
// implicit device synchronisation of cudaMalloc/cudaFree is not acceptable.
// This file gives them fp8_quantize_pertensor_static, which keeps the scratch
// in a file-scope __device__ array instead.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kernels.h"
#include "sp24.h"

namespace {

// Scratch of the static-scratch entry point.  Every GPU that loads the
// library holds these bytes until the process exits.
constexpr size_t kStaticScratchBytes = 256;
static_assert(sp24::kAmaxWorkspaceBytes <= kStaticScratchBytes, "static scratch too small");
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices];  // device address of g_static_scratch, per device

// In host code `g_static_scratch` only names a host-side stand-in; the
// device address must be looked up once per device with that device current.
cudaError_t scratch_address(int dev, void **out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

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
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SP24_ERR_ARCH;
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0) return SP24_ERR_ARCH;
  void *scratch = nullptr;
  cudaError_t e = scratch_address(dev, &scratch);
  if (e != cudaSuccess) {
    sp24::set_last_cuda_error(static_cast<int>(e));
    return SP24_ERR_CUDA;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left: clear the counters.
  e = cudaMemsetAsync(scratch, 0, sp24::kAmaxWorkspaceBytes, st);
  const int64_t nelem = rows * cols;
  if (e == cudaSuccess)
    e = sp24::launch_quantize_fused(X, nelem, static_cast<uint32_t *>(scratch), scale, q, status,
                                    sms, st);
  if (e != cudaSuccess) {
    sp24::set_last_cuda_error(static_cast<int>(e));
    return SP24_ERR_CUDA;
  }
  return SP24_OK;
}
