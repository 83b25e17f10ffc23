// Internal declarations shared by the library's translation units (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/gptq.h"

namespace gptq {

// Number of SMs of the current device (cached per device ordinal).
int num_sms();

// Builds a 2-D tiled TMA descriptor (dim 0 innermost) through the driver entry point.
gptq_status encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                           int elem_bytes, uint64_t dim0, uint64_t dim1, uint64_t ld_elems,
                           uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle);

// S1
gptq_status launch_hessian_bf16(float* S, int64_t cols, const void* X, int64_t n_tokens,
                                int64_t ldx, int32_t* info, cudaStream_t stream);
gptq_status launch_hessian_f32(float* S, int64_t cols, const float* X, int64_t n_tokens,
                               int64_t ldx, cudaStream_t stream);

// General fp32 matrix product on one tile grid:
//   C[m][n] = beta * C[m][n] + alpha * sum_{k = klo(m0, n0)}^{K-1} opA[m][k] * opB[k][n]
// opA[m][k] = transA ? A[k * lda + m] : A[m * lda + k]; opB likewise with B. With `lower`, output
// tiles lying entirely above the diagonal m == n are skipped. klo = max(0, m0 if klo_from_m,
// n0 if klo_from_n) where m0/n0 are the tile's first row/column (skips known-zero triangles).
struct GemmArgs {
  const float* A;
  int64_t lda;
  int transA;
  const float* B;
  int64_t ldb;
  int transB;
  float* C;
  int64_t ldc;
  int M, N, K;
  float alpha, beta;
  int lower;
  int klo_from_m;
  int klo_from_n;
};
gptq_status launch_gemm_f32(const GemmArgs& g, cudaStream_t stream);

// S2-S5
size_t prepare_workspace_bytes(int64_t cols);
gptq_status run_prepare_hinv(float* S_H, float* R, int64_t cols, int64_t n_total, float damp_rel,
                             void* ws, int32_t* info, cudaStream_t stream);

// S6-S8
size_t quantize_workspace_bytes(int64_t rows, int64_t cols, int block);
gptq_status run_quantize_layer(const void* W, gptq_dtype w_dtype, int64_t rows, int64_t cols,
                               int64_t ldw, const float* R, int bits, int group, int block,
                               float* W_hat, uint8_t* codes, float* scales, uint8_t* zeros,
                               float* err_sq, void* ws, int32_t* info, cudaStream_t stream);

// Host-side count of kernels this library has enqueued (diagnostic, see gptq_kernel_launches).
void count_launch(uint64_t n = 1);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace gptq
