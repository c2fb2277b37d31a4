// api.cu -- the extern "C" entry points declared in include/sp24.h: argument
// validation on the host, workspace bookkeeping and kernel launches.
#include <cuda_runtime.h>
#include <stdint.h>

#include "fp4_kernels.h"
#include "int8_kernels.h"
#include "kernels.h"
#include "sp24.h"

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 not sm_100

// SM count of the current device, or -1 when the device is not sm_100.
int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    g_sm_count[dev] = sms;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_arch_ok[dev] == 1 ? g_sm_count[dev] : -1;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SP24_OK;
  g_last_cuda_error = static_cast<int>(e);
  return SP24_ERR_CUDA;
}

// The single-launch kernels keep their amax counters in the workspace.
int check_workspace(const void *workspace, size_t ws_bytes) {
  if (!workspace || ws_bytes < sp24::kAmaxWorkspaceBytes) return SP24_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return SP24_ERR_ALIGN;
  return SP24_OK;
}

}  // namespace

void sp24::set_last_cuda_error(int e) { g_last_cuda_error = e; }
namespace sp24 {
// SM count of the current device for the other translation units (noalloc.cu)
int current_device_sm_count() { return device_sm_count(); }
}  // namespace sp24

extern "C" {

const char *sp24_version(void) { return "sp24 0.1 (sm_100a)"; }

int sp24_last_cuda_error(void) { return g_last_cuda_error; }

const char *sp24_status_str(int code) {
  switch (code) {
    case SP24_OK: return "ok";
    case SP24_ERR_NULL: return "a required pointer is NULL";
    case SP24_ERR_SHAPE: return "a dimension breaks the shape rules of the call";
    case SP24_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case SP24_ERR_DTYPE: return "unknown dtype";
    case SP24_ERR_CUDA: return "CUDA error (see sp24_last_cuda_error)";
    case SP24_ERR_WORKSPACE: return "workspace missing or too small";
    case SP24_ERR_ARCH: return "the current device is not sm_100 (B200)";
    default: return "unknown status";
  }
}

size_t sp24_workspace_size(int op, int64_t M, int64_t N, int64_t K, int dtype) {
  switch (op) {
    case SP24_OP_QUANTIZE:
    case SP24_OP_PRUNE_COMPRESS:
    case SP24_OP_SLIDE68_DECOMPOSE:
    case SP24_OP_SLIDE68_LIFT:
      return sp24::kAmaxWorkspaceBytes;
    case SP24_OP_QUANTIZE_GEMM_PACKED:
    case SP24_OP_LIFT_GEMM_PACKED: {
      // counters of the fused quantisation, then the GEMM's own workspace
      const int64_t Kg = op == SP24_OP_LIFT_GEMM_PACKED ? K / 2 * 3 : K;
      if (M < 1 || N < 128 || Kg < 128 || M > INT32_MAX || N > INT32_MAX || Kg > INT32_MAX) return 0;
      int sms = device_sm_count();
      if (sms <= 0) sms = 148;
      // the GEMM the call runs: the packed kind for the one-launch form, else
      // the kind sp24_gemm_packed takes for the shape
      const sp24::GemmKind gk = M * K / 8 <= sp24::kFusedXVec
                                    ? sp24::kSparseE4M3Packed
                                    : sp24::packed_kind(static_cast<int>(M), static_cast<int>(N), static_cast<int>(Kg), sms);
      return sp24::kFusedCounterBytes +
             sp24::plan_gemm(gk, static_cast<int>(M), static_cast<int>(N), static_cast<int>(Kg), sms).workspace_bytes();
    }
    case SP24_OP_GEMM_FP4: {
      if (M < 1 || N < 128 || K < 256 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return 0;
      int sms = device_sm_count();
      if (sms <= 0) sms = 148;
      return sp24::plan_gemm(sp24::kSparseFP4, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), sms)
          .workspace_bytes();
    }
    case SP24_OP_GEMM:
    case SP24_OP_GEMM_PACKED:
    case SP24_OP_GEMM_DENSE: {
      if (M < 1 || N < 128 || K < 128 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return 0;
      int sms = device_sm_count();
      if (sms <= 0) sms = 148;
      const sp24::GemmKind kind =
          op == SP24_OP_GEMM_DENSE ? sp24::kDenseE4M3
          : op == SP24_OP_GEMM_PACKED
              ? sp24::packed_kind(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), sms)
              : (dtype == SP24_DTYPE_BF16 ? sp24::kSparseBF16 : sp24::kSparseE4M3);
      return sp24::plan_gemm(kind, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), sms)
          .workspace_bytes();
    }
    default:
      return 0;
  }
}

int sp24_prune_compress(const void *W, int N, int K, int out_dtype, void *values, uint8_t *meta,
                        float *w_scale, void *pruned_dense, void *workspace, size_t ws_bytes,
                        int32_t *status, sp24_stream_t stream) {
  if (out_dtype != SP24_DTYPE_E4M3 && out_dtype != SP24_DTYPE_BF16) return SP24_ERR_DTYPE;
  if (!W || !values || !meta) return SP24_ERR_NULL;
  if (out_dtype == SP24_DTYPE_E4M3 && !w_scale) return SP24_ERR_NULL;
  if (N < 1 || K < 8 || K % 8 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta) ||
      (pruned_dense && !aligned16(pruned_dense)))
    return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nelem = static_cast<int64_t>(N) * K;
  const bool fp8 = out_dtype == SP24_DTYPE_E4M3;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  return cuda_status(sp24::launch_prune24_fused(W, nelem, fp8, static_cast<uint32_t *>(workspace),
                                                fp8 ? w_scale : nullptr, values, meta, pruned_dense,
                                                status, sms, st));
}

int sp24_prune_compress_packed(const void *W, int N, int K, void *packed, float *w_scale,
                               void *workspace, size_t ws_bytes, int32_t *status,
                               sp24_stream_t stream) {
  if (!W || !packed || !w_scale) return SP24_ERR_NULL;
  if (N < 128 || K < 128 || N % 128 != 0 || K % 128 != 0 ||
      static_cast<int64_t>(N) * K > (static_cast<int64_t>(1) << 38))
    return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  return cuda_status(sp24::launch_prune24_packed_fused(W, N, K, static_cast<uint32_t *>(workspace),
                                                       w_scale, static_cast<uint8_t *>(packed), status,
                                                       sms, reinterpret_cast<cudaStream_t>(stream)));
}

int slide68_decompose_packed(const void *W, int N, int K, void *packed, float *w_scale,
                             void *workspace, size_t ws_bytes, int32_t *status,
                             sp24_stream_t stream) {
  if (!W || !packed || !w_scale) return SP24_ERR_NULL;
  if (N < 128 || K < 256 || N % 128 != 0 || K % 256 != 0 ||
      static_cast<int64_t>(N) * K > (static_cast<int64_t>(1) << 38))
    return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  return cuda_status(sp24::launch_slide68_packed_fused(W, N, K, static_cast<uint32_t *>(workspace),
                                                       w_scale, static_cast<uint8_t *>(packed), status,
                                                       sms, reinterpret_cast<cudaStream_t>(stream)));
}

int fp8_quantize_pertensor(const void *X, int64_t rows, int64_t cols, uint8_t *q, float *scale,
                           void *workspace, size_t ws_bytes, int32_t *status,
                           sp24_stream_t stream) {
  if (!X || !q || !scale) return SP24_ERR_NULL;
  if (rows < 1 || cols < 1 || cols % 16 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(q)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nelem = rows * cols;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  if (sp24::small_quantize_fits(nelem))
    return cuda_status(sp24::launch_quantize_small(X, nelem, sp24::kSmallE4M3, scale, q, status, st));
  return cuda_status(sp24::launch_quantize_fused(X, nelem, static_cast<uint32_t *>(workspace), scale,
                                                 q, status, sms, st));
}

int int8_quantize_pertensor(const void *X, int64_t rows, int64_t cols, int8_t *q, float *scale, void *workspace,
                            size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (!X || !q || !scale) return SP24_ERR_NULL;
  if (rows < 1 || cols < 1 || cols % 16 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(q)) return SP24_ERR_ALIGN;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  if (sp24::small_quantize_fits(rows * cols))
    return cuda_status(sp24::launch_quantize_small(X, rows * cols, sp24::kSmallInt8, scale,
                                                   reinterpret_cast<uint8_t *>(q), status,
                                                   reinterpret_cast<cudaStream_t>(stream)));
  return cuda_status(sp24::launch_int8_quantize(X, rows * cols, static_cast<uint32_t *>(workspace), scale, q,
                                                status, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_prune_compress_int8(const void *W, int N, int K, int8_t *values, uint8_t *meta, float *w_scale,
                             void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (!W || !values || !meta || !w_scale) return SP24_ERR_NULL;
  if (N < 1 || K < 8 || K % 8 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta)) return SP24_ERR_ALIGN;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_int8_prune24(W, static_cast<int64_t>(N) * K, static_cast<uint32_t *>(workspace),
                                               w_scale, values, meta, status, sms,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int slide68_decompose(const void *W, int N, int K, int out_dtype, void *values, uint8_t *meta,
                      float *w_scale, void *workspace, size_t ws_bytes, int32_t *status,
                      sp24_stream_t stream) {
  if (out_dtype != SP24_DTYPE_E4M3 && out_dtype != SP24_DTYPE_BF16) return SP24_ERR_DTYPE;
  if (!W || !values || !meta) return SP24_ERR_NULL;
  if (out_dtype == SP24_DTYPE_E4M3 && !w_scale) return SP24_ERR_NULL;
  if (N < 1 || K < 16 || K % 16 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nelem = static_cast<int64_t>(N) * K;
  const bool fp8 = out_dtype == SP24_DTYPE_E4M3;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  return cuda_status(sp24::launch_slide68_fused(W, nelem, fp8, static_cast<uint32_t *>(workspace),
                                                fp8 ? w_scale : nullptr, values, meta, status, sms,
                                                st));
}

int slide68_lift(const void *X, int M, int K, uint8_t *q_lifted, float *scale, void *workspace,
                 size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (!X || !q_lifted || !scale) return SP24_ERR_NULL;
  if (M < 1 || K < 16 || K % 16 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(q_lifted)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nelem = static_cast<int64_t>(M) * K;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  if (sp24::small_quantize_fits(nelem))
    return cuda_status(sp24::launch_quantize_small(X, nelem, sp24::kSmallLift, scale, q_lifted, status, st));
  return cuda_status(sp24::launch_lift_fused(X, nelem, static_cast<uint32_t *>(workspace), scale,
                                             q_lifted, status, sms, st));
}

static int gemm_common(sp24::GemmKind kind, const void *Xq, const float *x_scale,
                       const void *w_values, const uint8_t *w_meta, const float *w_scale, void *Y,
                       int M, int N, int K, void *workspace, size_t ws_bytes, int32_t *status,
                       sp24_stream_t stream) {
  const bool sparse = kind != sp24::kDenseE4M3 && kind != sp24::kSparseE4M3Packed && kind != sp24::kSparseI8Packed;
  if (!Xq || !w_values || !Y || (sparse && !w_meta)) return SP24_ERR_NULL;
  const int kmod = 128;
  if (M < 1 || N < 128 || N % 128 != 0 || K < kmod || K % kmod != 0) return SP24_ERR_SHAPE;
  if (!aligned16(Xq) || !aligned16(w_values) || !aligned16(Y) || (sparse && !aligned16(w_meta)))
    return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  if (kind == sp24::kSparseE4M3Packed) kind = sp24::packed_kind(M, N, K, sms);
  const sp24::GemmPlan pl = sp24::plan_gemm(kind, M, N, K, sms);
  if (pl.workspace_bytes() > 0) {
    if (!workspace || ws_bytes < pl.workspace_bytes()) return SP24_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SP24_ERR_ALIGN;
  }
  return cuda_status(sp24::launch_gemm(kind, pl, Xq, x_scale, w_values, w_meta, w_scale, Y, M, N, K,
                                       workspace, status, reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_gemm(const void *Xq, const float *x_scale, const void *w_values, const uint8_t *w_meta,
              const float *w_scale, void *Y, int M, int N, int K, int dtype, void *workspace,
              size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (dtype == SP24_DTYPE_E4M3)
    return gemm_common(sp24::kSparseE4M3, Xq, x_scale, w_values, w_meta, w_scale, Y, M, N, K,
                       workspace, ws_bytes, status, stream);
  if (dtype == SP24_DTYPE_BF16)
    return gemm_common(sp24::kSparseBF16, Xq, nullptr, w_values, w_meta, nullptr, Y, M, N, K,
                       workspace, ws_bytes, status, stream);
  return SP24_ERR_DTYPE;
}

int sp24_pack_weights(const uint8_t *values, const uint8_t *meta, int N, int K, void *packed,
                      sp24_stream_t stream) {
  if (!values || !meta || !packed) return SP24_ERR_NULL;
  if (N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(values) || !aligned16(meta) || !aligned16(packed)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_pack_weights(values, meta, N, K, static_cast<uint8_t *>(packed), sms,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_gemm_packed(const void *Xq, const float *x_scale, const void *packed, const float *w_scale,
                     void *Y, int M, int N, int K, void *workspace, size_t ws_bytes, int32_t *status,
                     sp24_stream_t stream) {
  return gemm_common(sp24::kSparseE4M3Packed, Xq, x_scale, packed, nullptr, w_scale, Y, M, N, K,
                     workspace, ws_bytes, status, stream);
}

int fp4_quantize_pertensor(const void *X, int64_t rows, int64_t cols, uint8_t *q, float *scale, void *workspace,
                           size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (!X || !q || !scale) return SP24_ERR_NULL;
  if (rows < 1 || cols < 1 || cols % 32 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(q)) return SP24_ERR_ALIGN;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  if (sp24::small_quantize_fits(rows * cols))
    return cuda_status(sp24::launch_quantize_small(X, rows * cols, sp24::kSmallFp4, scale, q, status,
                                                   reinterpret_cast<cudaStream_t>(stream)));
  return cuda_status(sp24::launch_fp4_quantize(X, rows * cols, static_cast<uint32_t *>(workspace), scale, q,
                                               status, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_prune_compress_fp4(const void *W, int N, int K, uint8_t *values, uint8_t *meta, float *w_scale,
                            void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (!W || !values || !meta || !w_scale) return SP24_ERR_NULL;
  if (N < 1 || K < 64 || K % 64 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta)) return SP24_ERR_ALIGN;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_fp4_prune24(W, static_cast<int64_t>(N) * K, static_cast<uint32_t *>(workspace),
                                              w_scale, values, meta, status, sms,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_gemm_fp4(const uint8_t *Xq, const float *x_scale, const uint8_t *w_values, const uint8_t *w_meta,
                  const float *w_scale, void *Y, int M, int N, int K, void *workspace, size_t ws_bytes,
                  int32_t *status, sp24_stream_t stream) {
  if (!Xq || !w_values || !w_meta || !Y) return SP24_ERR_NULL;
  if (M < 1 || N < 128 || N % 128 != 0 || K < 256 || K % 256 != 0) return SP24_ERR_SHAPE;
  // the 4-bit tensor maps want 32-byte aligned bases
  if ((reinterpret_cast<uintptr_t>(Xq) & 31u) || (reinterpret_cast<uintptr_t>(w_values) & 31u) ||
      !aligned16(w_meta) || !aligned16(Y))
    return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  const sp24::GemmPlan pl = sp24::plan_gemm(sp24::kSparseFP4, M, N, K, sms);
  if (pl.workspace_bytes() > 0) {
    if (!workspace || ws_bytes < pl.workspace_bytes()) return SP24_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SP24_ERR_ALIGN;
  }
  return cuda_status(sp24::launch_gemm(sp24::kSparseFP4, pl, Xq, x_scale, w_values, w_meta, w_scale, Y, M, N, K,
                                       workspace, status, reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_gemm_int8_packed(const int8_t *Xq, const float *x_scale, const void *packed, const float *w_scale,
                          void *Y, int M, int N, int K, void *workspace, size_t ws_bytes, int32_t *status,
                          sp24_stream_t stream) {
  return gemm_common(sp24::kSparseI8Packed, Xq, x_scale, packed, nullptr, w_scale, Y, M, N, K, workspace,
                     ws_bytes, status, stream);
}

static int quant_gemm_common(bool lift, const void *X, int M, int N, int K, const void *packed,
                             const float *w_scale, uint8_t *Xq, float *x_scale, void *Y,
                             void *workspace, size_t ws_bytes, int32_t *status,
                             sp24_stream_t stream) {
  if (!X || !packed || !Xq || !x_scale || !Y) return SP24_ERR_NULL;
  if (M < 1 || M > 256 || N < 128 || N % 128 != 0 || K < 128 || K % (lift ? 256 : 128) != 0)
    return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(packed) || !aligned16(Xq) || !aligned16(Y)) return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  const int Kg = lift ? K / 2 * 3 : K;
  const int64_t nelem = static_cast<int64_t>(M) * K;
  const bool one_launch = nelem / 8 <= sp24::kFusedXVec;
  // above the one-launch size: the GEMM sp24_gemm_packed runs for the shape
  // (the same kind, so the same Y bit for bit)
  const sp24::GemmKind gk = one_launch ? sp24::kSparseE4M3Packed : sp24::packed_kind(M, N, Kg, sms);
  const sp24::GemmPlan pl = sp24::plan_gemm(gk, M, N, Kg, sms);
  if (!workspace || ws_bytes < sp24::kFusedCounterBytes + pl.workspace_bytes()) return SP24_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SP24_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void *gemm_ws = static_cast<uint8_t *>(workspace) + sp24::kFusedCounterBytes;
  if (one_launch) {
    // one launch: every CTA quantises all of X in front of its GEMM tiles
    sp24::GemmFusedX fx;
    fx.x = X;
    fx.lift = lift ? 1 : 0;
    fx.xq = Xq;
    fx.x_scale = x_scale;
    return cuda_status(sp24::launch_gemm_quant(pl, fx, packed, w_scale, Y, M, N, Kg, gemm_ws, status, st));
  }
  // Larger X: the quantiser (one cluster for decode-sized X, which lets the
  // GEMM launch at once and stream its weights meanwhile; the streamed
  // kernel beyond that), then the GEMM on its codes.
  cudaError_t e;
  if (sp24::small_quantize_fits(nelem))
    e = sp24::launch_quantize_small(X, nelem, lift ? sp24::kSmallLift : sp24::kSmallE4M3, x_scale, Xq, status, st);
  else if (lift)
    e = sp24::launch_lift_fused(X, nelem, static_cast<uint32_t *>(workspace), x_scale, Xq, status, sms, st);
  else
    e = sp24::launch_quantize_fused(X, nelem, static_cast<uint32_t *>(workspace), x_scale, Xq, status, sms, st);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(sp24::launch_gemm(gk, pl, Xq, x_scale, packed, nullptr, w_scale, Y, M, N, Kg, gemm_ws, status,
                                       st));
}

int sp24_quantize_gemm_packed(const void *X, int M, int N, int K, const void *packed,
                              const float *w_scale, uint8_t *Xq, float *x_scale, void *Y,
                              void *workspace, size_t ws_bytes, int32_t *status,
                              sp24_stream_t stream) {
  return quant_gemm_common(false, X, M, N, K, packed, w_scale, Xq, x_scale, Y, workspace, ws_bytes,
                           status, stream);
}

int slide68_lift_gemm_packed(const void *X, int M, int N, int K, const void *packed,
                             const float *w_scale, uint8_t *Xq_lifted, float *x_scale, void *Y,
                             void *workspace, size_t ws_bytes, int32_t *status,
                             sp24_stream_t stream) {
  return quant_gemm_common(true, X, M, N, K, packed, w_scale, Xq_lifted, x_scale, Y, workspace,
                           ws_bytes, status, stream);
}

// K' = K (2n - 2) / n for the (2n-2):2n decomposition; 0 when K does not fit.
static int64_t slide_kprime(int64_t K, int n) {
  if (n < 3 || n > 5 || K % (2 * n) != 0) return 0;
  const int64_t kp = K / (2 * n) * 4 * (n - 1);
  return kp % 16 == 0 ? kp : 0;
}

int slide_decompose(const void *W, int N, int K, int n, uint8_t *values, uint8_t *meta, float *w_scale,
                    void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (n == 4) return slide68_decompose(W, N, K, SP24_DTYPE_E4M3, values, meta, w_scale, workspace, ws_bytes,
                                       status, stream);
  if (!W || !values || !meta || !w_scale) return SP24_ERR_NULL;
  if (N < 1 || slide_kprime(K, n) == 0 || (static_cast<int64_t>(N) * K) % 8 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta) || !aligned16(w_scale)) return SP24_ERR_ALIGN;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_slide_decompose(W, N, K, n, static_cast<uint32_t *>(workspace), w_scale, values,
                                                  meta, status, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int slide_lift(const void *X, int M, int K, int n, uint8_t *q_lifted, float *scale, void *workspace,
               size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (n == 4) return slide68_lift(X, M, K, q_lifted, scale, workspace, ws_bytes, status, stream);
  if (!X || !q_lifted || !scale) return SP24_ERR_NULL;
  if (M < 1 || slide_kprime(K, n) == 0 || (static_cast<int64_t>(M) * K) % 8 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(q_lifted) || !aligned16(scale)) return SP24_ERR_ALIGN;
  const int rc = check_workspace(workspace, ws_bytes);
  if (rc != SP24_OK) return rc;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_slide_lift(X, M, K, n, static_cast<uint32_t *>(workspace), scale, q_lifted,
                                             status, sms, reinterpret_cast<cudaStream_t>(stream)));
}

int fp8_quantize_pertoken(const void *X, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                          int32_t *status, sp24_stream_t stream) {
  if (!X || !q || !scales) return SP24_ERR_NULL;
  if (rows < 1 || cols < 8 || cols % 8 != 0 || rows > INT32_MAX * 8ll) return SP24_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(q) || !aligned16(scales)) return SP24_ERR_ALIGN;
  if (device_sm_count() < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_quantize_pertoken(X, rows, cols, q, scales, status,
                                                    reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_prune_compress_perchannel(const void *W, int N, int K, uint8_t *values, uint8_t *meta,
                                   float *w_scales, int32_t *status, sp24_stream_t stream) {
  if (!W || !values || !meta || !w_scales) return SP24_ERR_NULL;
  if (N < 1 || K < 8 || K % 8 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(values) || !aligned16(meta) || !aligned16(w_scales)) return SP24_ERR_ALIGN;
  if (device_sm_count() < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_prune24_perchannel(W, N, K, values, meta, w_scales, status,
                                                     reinterpret_cast<cudaStream_t>(stream)));
}

int sp24_gemm_packed_scaled(const void *Xq, const float *x_scales, int x_per_token, const void *packed,
                            const float *w_scales, int w_per_channel, void *Y, int M, int N, int K,
                            void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  if (!Xq || !x_scales || !packed || !w_scales || !Y) return SP24_ERR_NULL;
  if (M < 1 || N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0) return SP24_ERR_SHAPE;
  if (!aligned16(Xq) || !aligned16(packed) || !aligned16(Y) || !aligned16(x_scales) || !aligned16(w_scales))
    return SP24_ERR_ALIGN;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  // the tiles sp24_gemm_packed takes for the shape (SM pairs included)
  const sp24::GemmPlan pl = sp24::plan_gemm(sp24::packed_kind(M, N, K, sms), M, N, K, sms);
  if (pl.workspace_bytes() > 0) {
    if (!workspace || ws_bytes < pl.workspace_bytes()) return SP24_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SP24_ERR_ALIGN;
  }
  return cuda_status(sp24::launch_gemm_scaled(pl, Xq, x_scales, x_per_token ? 1 : 0, packed, w_scales,
                                              w_per_channel ? 1 : 0, Y, M, N, K, workspace, status,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

int fp8_gemm_dense(const uint8_t *Xq, const float *x_scale, const uint8_t *Wq,
                   const float *w_scale, void *Y, int M, int N, int K, void *workspace,
                   size_t ws_bytes, int32_t *status, sp24_stream_t stream) {
  return gemm_common(sp24::kDenseE4M3, Xq, x_scale, Wq, nullptr, w_scale, Y, M, N, K, workspace,
                     ws_bytes, status, stream);
}

int sp24_debug_e4m3_encode(const float *v, uint8_t *out, int64_t n, sp24_stream_t stream) {
  if (n < 0) return SP24_ERR_SHAPE;
  if (n > 0 && (!v || !out)) return SP24_ERR_NULL;
  const int sms = device_sm_count();
  if (sms < 0) return SP24_ERR_ARCH;
  return cuda_status(sp24::launch_e4m3_encode(v, out, n, sms, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
