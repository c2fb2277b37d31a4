// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernels (elementwise.cu, gemm.cu, stream.cu).  Not installed; not part of
// the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sp24 {

// 2-D tiled TMA descriptor of a row-major [outer, inner] tensor of
// elem_bytes-sized elements (row pitch inner * elem_bytes), box
// [box_outer, box_inner].  False when the driver entry point is missing or
// the encoder rejects the arguments.
bool make_tensor_map_2d(CUtensorMap *map, const void *ptr, CUtensorMapDataType dt, int elem_bytes,
                        uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle sw);

// ---- elementwise.cu
cudaError_t launch_e4m3_encode(const float *v, uint8_t *out, int64_t n, int sm_count,
                               cudaStream_t st);
// Re-lay 2:4 E4M3 weights (canonical values + metadata) into the GEMM's
// tile-packed layout: one 10240-byte block per (128-row tile, 128-K block).
cudaError_t launch_pack_weights(const uint8_t *values, const uint8_t *meta, int N, int K,
                                uint8_t *packed, int sm_count, cudaStream_t st);
constexpr int kPackedBlockBytes = 128 * 64 + 128 * 16;

// ---- stream.cu: single-launch TMA-streamed kernels (cooperative grid).
// `ws` must hold kAmaxWorkspaceBytes of zeroed counters; they are zero again
// when the kernel ends.
cudaError_t launch_quantize_fused(const void *x, int64_t nelem, uint32_t *ws, float *scale,
                                  uint8_t *q, int32_t *status, int sm_count, cudaStream_t st);
cudaError_t launch_lift_fused(const void *x, int64_t nelem, uint32_t *ws, float *scale,
                              uint8_t *q, int32_t *status, int sm_count, cudaStream_t st);
cudaError_t launch_prune24_fused(const void *w, int64_t nelem, bool fp8, uint32_t *ws,
                                 float *scale, void *values, uint8_t *meta, void *dense,
                                 int32_t *status, int sm_count, cudaStream_t st);
// 2:4 prune + E4M3 quantise written straight into the tile-packed layout
// (N % 128 == 0, K % 128 == 0).
cudaError_t launch_prune24_packed_fused(const void *w, int N, int K, uint32_t *ws, float *scale,
                                        uint8_t *packed, int32_t *status, int sm_count,
                                        cudaStream_t st);
// 6:8 decomposition + E4M3 quantise written straight into the tile-packed
// layout of the lifted 2:4 operand (N % 128 == 0, K % 256 == 0).
cudaError_t launch_slide68_packed_fused(const void *w, int N, int K, uint32_t *ws, float *scale,
                                        uint8_t *packed, int32_t *status, int sm_count,
                                        cudaStream_t st);
cudaError_t launch_slide68_fused(const void *w, int64_t nelem, bool fp8, uint32_t *ws,
                                 float *scale, void *values, uint8_t *meta, int32_t *status,
                                 int sm_count, cudaStream_t st);

// ---- rowscale.cu: per-token / per-channel scales (one warp per row).
cudaError_t launch_quantize_pertoken(const void *x, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                                     int32_t *status, cudaStream_t st);
cudaError_t launch_prune24_perchannel(const void *w, int N, int K, uint8_t *values, uint8_t *meta,
                                      float *scales, int32_t *status, cudaStream_t st);

// ---- slide.cu: general (2N-2):2N (N = 3, 5); `ws` as for the streamed kernels.
cudaError_t launch_slide_decompose(const void *w, int N, int K, int n, uint32_t *ws, float *scale,
                                   uint8_t *values, uint8_t *meta, int32_t *status, int sms, cudaStream_t st);
cudaError_t launch_slide_lift(const void *x, int M, int K, int n, uint32_t *ws, float *scale, uint8_t *q,
                              int32_t *status, int sms, cudaStream_t st);

// Records the CUDA error reported by sp24_last_cuda_error() (api.cu).
void set_last_cuda_error(int e);

// Bytes of scratch the amax/scale reduction uses (two counters, padded).
constexpr size_t kAmaxWorkspaceBytes = 256;

// Prefix of the fused quantise + GEMM workspace: the counters of the
// activation quantiser that runs in front of the GEMM when X is too large for
// the one-launch form (kAmaxWorkspaceBytes used, the rest reserved).  Zero
// before the first call and after every call.
constexpr size_t kFusedCounterBytes = 8192;

// ---- smallx.cu: decode-sized activations (at most kSmallXVec 8-element
// vectors, nelem % 8 == 0) quantised by one thread-block cluster, no
// workspace: E4M3 codes [nelem], their 6:8 lift (rows of 16k elements)
// [3 nelem / 2], INT8 codes [nelem] or FP4 codes [nelem / 2] (two per byte).
constexpr int64_t kSmallXVec = 16384;
enum SmallEnc : int { kSmallE4M3 = 0, kSmallLift = 1, kSmallInt8 = 2, kSmallFp4 = 3 };
bool small_quantize_fits(int64_t nelem);
cudaError_t launch_quantize_small(const void *x, int64_t nelem, SmallEnc enc, float *scale, uint8_t *q,
                                  int32_t *status, cudaStream_t st);

// ---- gemm.cu
enum GemmKind : int {
  kSparseE4M3 = 0,
  kDenseE4M3 = 1,
  kSparseBF16 = 2,
  kSparseE4M3Packed = 3,
  kSparseI8Packed = 4,
  kSparseFP4 = 5,  // E2M1 codes, two per byte, canonical 2:4 layout; stages of 256 K
  kSparseE4M3Pair = 6  // the packed E4M3 kind on SM pairs (128- and 224-token tiles, N % 256 == 0)
};

// How a GEMM call is cut into CTAs: tile shape, work decomposition and the
// scratch a stream-K reduction needs.
constexpr size_t kGemmCounterBytes = 16384;  // tile counters: a fixed workspace prefix

struct GemmPlan {
  int bn;            // tokens per tile (MMA N)
  int mt;            // 128-row W tiles per CTA tile (1 or 2)
  int kb;            // 128-K blocks per pipeline stage (1 or 2)
  int bk;            // logical K per pipeline stage (128 kb)
  int tiles_n;       // N / (128 mt)
  int tiles_m;       // ceil(M / bn)
  int num_kb;        // K / bk
  int num_tiles;
  int64_t units;     // num_tiles * num_kb
  bool stream_k;     // some tiles are split over CTAs (needs the workspace)
  int grid;          // persistent CTAs (one per SM at most)
  int dp_tiles;      // tiles taken whole
  int sk_grid;       // CTAs sharing the leftover tiles' (tile, k-block) units
  int64_t sk_units;
  size_t partial_bytes;
  size_t counter_bytes;
  int pair;          // planned for kSparseE4M3Pair (grid counts CTAs: two per pair)
  size_t workspace_bytes() const { return stream_k ? counter_bytes + partial_bytes : 0; }
};

GemmPlan plan_gemm(GemmKind kind, int M, int N, int K, int sm_count);

// The kind the packed E4M3 GEMM runs as: kSparseE4M3Pair where N % 256 == 0,
// the device runs CTA pairs and the plan takes 224-token tiles of two weight
// row tiles (prefill) or 128-token tiles of 129..1023 tokens, else
// kSparseE4M3Packed.
GemmKind packed_kind(int M, int N, int K, int sm_count);

// Launch the tcgen05 GEMM.  `workspace` must hold plan.workspace_bytes()
// bytes whose counter prefix is zero (it is zero again afterwards).
cudaError_t launch_gemm(GemmKind kind, const GemmPlan &plan, const void *xq, const float *x_scale,
                        const void *w_values, const uint8_t *w_meta, const float *w_scale,
                        void *y, int M, int N, int K, void *workspace, int32_t *status,
                        cudaStream_t st);

// The packed E4M3 GEMM with scale vectors: x_scales holds M per-token scales
// when x_vec (else one), w_scales N per-channel scales when w_vec (else one).
cudaError_t launch_gemm_scaled(const GemmPlan &plan, const void *xq, const float *x_scales, int x_vec,
                               const void *packed, const float *w_scales, int w_vec, void *y, int M, int N,
                               int K, void *workspace, int32_t *status, cudaStream_t st);

// The packed E4M3 GEMM with the per-tensor quantisation of its activations
// fused in front, for X of at most kFusedXVec 8-element vectors (plan from
// plan_gemm(kSparseE4M3Packed, M, N, K); bn <= 128, mt == 1).  K is the
// GEMM's K: the columns of X, or 3/2 of them with lift.
constexpr int64_t kFusedXVec = 1024;
struct GemmFusedX {
  const void *x;       // bf16 [M, Kx]
  int lift;            // 0: codes [M, Kx]; 1: SlideSparse lift, codes [M, 3 Kx / 2]
  uint8_t *xq;         // out: the E4M3 codes (the GEMM's B operand)
  float *x_scale;      // out: amax|X| / 448 (1 when amax = 0)
};
cudaError_t launch_gemm_quant(const GemmPlan &plan, const GemmFusedX &fx, const void *packed,
                              const float *w_scale, void *y, int M, int N, int K, void *workspace,
                              int32_t *status, cudaStream_t st);

}  // namespace sp24
