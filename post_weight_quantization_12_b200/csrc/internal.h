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

// fp32-accurate matrix product on the tensor cores (3xTF32, see gemm_tc.cu):
//   C[m][n] = alpha * sum_{k = klo}^{K-1} opA[m][k] * opB[k][n] + beta * C[m][n]
// Each operand comes as its tf32 split (x_big, x_small), both with the same layout:
//   opA[m][k] = a_mn ? A[k * lda + m] : A[m * lda + k]
//   opB[k][n] = b_mn ? B[k * ldb + n] : B[n * ldb + k]
// With `lower`, 128 x 128 output tiles entirely above the diagonal m == n are skipped.
// klo = max(0, m0 if klo_from_m, n0 if klo_from_n) for the tile's first row m0 / column n0, and
// khi = min(K, m0 + 128 if khi_from_m), to skip known-zero triangles (m0, n0 are multiples of
// 128). C may be null (then beta must be 0); if Cbig is set, the tf32 split of the result is also
// written there (ld_split).
// Batches: `batch` independent products of the same shape whose operands and results sit
// bstride rows and bstride columns further along the same matrices (blocks along a diagonal);
// every coordinate of A, B, C and the split is shifted by b * bstride for batch b.
// Requirements: operand bases 16-byte aligned, lda % 4 == 0, ldb % 4 == 0.
struct TcGemmArgs {
  const float* Ab;
  const float* As;
  const float* Bb;
  const float* Bs;
  int64_t lda, ldb;
  int a_mn, b_mn;
  int M, N, K;
  float alpha, beta;
  int lower, klo_from_m, klo_from_n;
  float* C;
  int64_t ldc;
  float* Cbig;
  float* Csmall;
  int64_t ld_split;
  int32_t* info;
  int batch = 1;
  int64_t bstride = 0;
  int khi_from_m = 0;
};
gptq_status launch_gemm_tc(const TcGemmArgs& g, cudaStream_t stream);

// x -> (tf32(x), x - tf32(x)) for a rows x cols block.
gptq_status launch_split_tf32(const float* X, int64_t ldx, int64_t rows, int64_t cols, float* big,
                              float* small, int64_t ldo, cudaStream_t stream);

// S3/S5: steps 0 .. T-2 of the blocked Cholesky of A (n x n, n % 4 == 0, T = ceil(n / 128) >= 2)
// as fused launches (potrf_step.cu). On entry X_00's split is at (Vb, Vs) (block 0 of an n x n
// matrix with ld ld_dinv when per_block, else parity 0 of two stacked 128 x 128 blocks), the
// first panel's split at parity 0 of (Pb, Ps) (two stacked n x 128 buffers, absolute rows) and
// flags[0 .. T) is zero. Fills L's split (Lb, Ls; n x n), the inverses of the diagonal blocks,
// and, with store_l, L in A.
gptq_status launch_potrf_fused(float* A, int64_t n, float* Lb, float* Ls, float* Vb, float* Vs,
                               int64_t ld_dinv, bool per_block, float* Pb, float* Ps,
                               int32_t* flags, int32_t* info, int info_base, int rev_n,
                               bool store_l, cudaStream_t stream);

// S2-S5
size_t prepare_workspace_bytes(int64_t cols);
gptq_status run_prepare_hinv(float* S_H, float* R, int64_t cols, int64_t n_total, float damp_rel,
                             int route, void* ws, int32_t* info, cudaStream_t stream);

// S6-S8
size_t quantize_workspace_bytes(int64_t rows, int64_t cols, int block);
// Every argument check of gptq_quantize_layer except the workspace's (GPTQ_OK when they pass).
gptq_status check_quantize_args(const void* W, gptq_dtype w_dtype, int64_t rows, int64_t cols,
                                int64_t ldw, const float* R, int bits, int group, int block,
                                const float* W_hat, const uint8_t* codes, const float* scales,
                                const uint8_t* zeros);
gptq_status run_quantize_layer(const void* W, gptq_dtype w_dtype, int64_t rows, int64_t cols,
                               int64_t ldw, const float* R, int bits, int group, int block,
                               float* W_hat, uint8_t* codes, float* scales, uint8_t* zeros,
                               float* err_sq, void* ws, int32_t* info, cudaStream_t stream);

// Packed 4-bit codes and the W4A16 product (w4a16.cu).
gptq_status run_pack_codes_4bit(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldc,
                                uint32_t* packed, int32_t* info, cudaStream_t stream);
gptq_status run_pack_codes_3bit(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldc,
                                uint32_t* packed, int32_t* info, cudaStream_t stream);
// n > 16 activation rows: the tensor-core form of the same product (w4a16_gemm.cu).
gptq_status run_w4a16_gemm(const uint32_t* packed, const float* scales, const uint8_t* zeros,
                           int64_t rows, int64_t cols, int group, const void* x, int64_t n,
                           int64_t ldx, float* y, int64_t ldy, int32_t* info, cudaStream_t stream);
gptq_status run_w4a16_gemv(const uint32_t* packed, const float* scales, const uint8_t* zeros,
                           int64_t rows, int64_t cols, int group, const void* x, int64_t n,
                           int64_t ldx, float* y, int64_t ldy, int32_t* info, cudaStream_t stream);

// Randomized Hadamard rotation of the rows' input-channel axis (rotation.cu).
int hadamard_block_order(int64_t n);
gptq_status run_hadamard_rotate(const void* X, int x_bf16, int64_t ldx, int64_t rows, int64_t n,
                                const uint32_t* sign_bits, void* Y, int y_bf16, int64_t ldy,
                                cudaStream_t stream);

// OBQ greedy-order reference for layers of at most 128 columns (obq.cu).
gptq_status run_obq_quantize(const float* W, int64_t rows, int64_t cols, int64_t ldw,
                             const double* Hinv, int bits, int greedy, uint8_t* codes,
                             float* W_hat, int32_t* order, double* loss, float* scales,
                             uint8_t* zeros, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the current device. The
// attribute belongs to the (kernel, device) pair; each pair is set once, under a lock.
gptq_status set_max_dynamic_smem(const void* kernel, int bytes);

// Host-side count of kernels this library has enqueued (diagnostic, see gptq_kernel_launches).
void count_launch(uint64_t n = 1);

// Launch with programmatic stream serialization: the kernel may begin while the previous kernel
// in the stream drains; it must call griddep_wait() before touching global memory. Counts the
// launch and reports launch errors.
template <typename... KArgs, typename... Args>
inline gptq_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  count_launch();
  return e == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace gptq
