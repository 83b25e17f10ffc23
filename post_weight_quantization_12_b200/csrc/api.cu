// C ABI of libgptq_b200: argument validation and dispatch to the kernels (see include/gptq.h).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace gptq {

static std::atomic<uint64_t> g_launches{0};
void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// One CTA waits on a barrier that nothing arrives on; the bounded wait must give up and report.
__global__ void selftest_wait_kernel(int32_t* info, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, info, limit_ns);
  __syncthreads();
}

// One thread waits for a flag in global memory to reach 1; unless something sets it, the bounded
// wait must give up and report.
__global__ void selftest_flag_kernel(const int32_t* flag, int32_t* info, uint64_t limit_ns) {
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    flag_wait_bounded(flag, 1, &abort_flag, info, limit_ns);
  }
}

gptq_status set_max_dynamic_smem(const void* kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ECUDA;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;  // (kernel, device) -> bytes set
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({kernel, dev});
  if (it != done.end() && it->second >= bytes) return GPTQ_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return GPTQ_ECUDA;
  done[{kernel, dev}] = bytes;
  return GPTQ_OK;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

gptq_status encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                           int elem_bytes, uint64_t dim0, uint64_t dim1, uint64_t ld_elems,
                           uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return GPTQ_ECUDA;
  cuuint64_t dims[2] = {dim0, dim1};
  cuuint64_t strides[1] = {ld_elems * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_EINVAL;
}

}  // namespace gptq

using namespace gptq;

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

gptq_status gptq::check_quantize_args(const void* W, gptq_dtype w_dtype, int64_t rows,
                                      int64_t cols, int64_t ldw, const float* R, int bits,
                                      int group, int block, const float* W_hat,
                                      const uint8_t* codes, const float* scales,
                                      const uint8_t* zeros) {
  if (W == nullptr || R == nullptr || W_hat == nullptr || codes == nullptr || scales == nullptr ||
      zeros == nullptr)
    return GPTQ_EINVAL;
  if (rows <= 0 || cols <= 0 || ldw < cols) return GPTQ_EINVAL;
  if (cols % 4 != 0 || !aligned(R, 16) || !aligned(W_hat, 16)) return GPTQ_EINVAL;
  if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_FP32) return GPTQ_EINVAL;
  if (bits < 2 || bits > 8) return GPTQ_EINVAL;
  if (block != 32 && block != 64 && block != 128) return GPTQ_EINVAL;
  if (group == 0 || group < -1) return GPTQ_EINVAL;
  if (group > 0 && (cols % group != 0 || !(group % block == 0 || block % group == 0)))
    return GPTQ_EINVAL;
  if (cols > 65536 || rows > (static_cast<int64_t>(1) << 30) ||
      rows * cols > (static_cast<int64_t>(1) << 40))
    return GPTQ_EUNSUPPORTED;
  return GPTQ_OK;
}

extern "C" {

gptq_status gptq_hessian_accumulate(float* S_dev, int64_t cols, const void* X_dev,
                                    gptq_dtype x_dtype, int64_t n_tokens, int64_t ldx,
                                    int32_t* info_dev, void* stream) {
  if (S_dev == nullptr || cols <= 0 || n_tokens < 0 || ldx < cols) return GPTQ_EINVAL;
  if (cols > (1 << 20)) return GPTQ_EUNSUPPORTED;
  if (n_tokens == 0) return GPTQ_OK;
  if (X_dev == nullptr) return GPTQ_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (x_dtype == GPTQ_BF16) {
    if (cols % 8 != 0 || ldx % 8 != 0 || !aligned(X_dev, 16) || !aligned(S_dev, 16))
      return GPTQ_EINVAL;
    if (n_tokens > (static_cast<int64_t>(1) << 31) - 64) return GPTQ_EUNSUPPORTED;
    return launch_hessian_bf16(S_dev, cols, X_dev, n_tokens, ldx, info_dev, s);
  }
  if (x_dtype == GPTQ_FP32) {
    if (!aligned(X_dev, 4)) return GPTQ_EINVAL;
    return launch_hessian_f32(S_dev, cols, static_cast<const float*>(X_dev), n_tokens, ldx, s);
  }
  return GPTQ_EINVAL;
}

gptq_status gptq_prepare_hinv(float* S_H_dev, float* R_dev, int64_t cols, int64_t n_total,
                              float damp_rel, void* ws_dev, size_t ws_bytes, int32_t* info_dev,
                              void* stream) {
  return gptq_prepare_hinv_route(S_H_dev, R_dev, cols, n_total, damp_rel, GPTQ_ROUTE_DEFAULT,
                                 ws_dev, ws_bytes, info_dev, stream);
}

gptq_status gptq_prepare_hinv_route(float* S_H_dev, float* R_dev, int64_t cols, int64_t n_total,
                                    float damp_rel, int route, void* ws_dev, size_t ws_bytes,
                                    int32_t* info_dev, void* stream) {
  if (route != GPTQ_ROUTE_DEFAULT && route != GPTQ_ROUTE_THREE_STEP && route != GPTQ_ROUTE_REVERSED)
    return GPTQ_EINVAL;
  if (S_H_dev == nullptr || R_dev == nullptr || cols <= 0 || n_total <= 0) return GPTQ_EINVAL;
  if (cols % 4 != 0 || !aligned(S_H_dev, 16) || !aligned(R_dev, 16)) return GPTQ_EINVAL;
  if (!(damp_rel >= 0.f) || !(damp_rel < 1e30f)) return GPTQ_EINVAL;
  if (cols > 65536) return GPTQ_EUNSUPPORTED;
  if (ws_dev == nullptr || ws_bytes < prepare_workspace_bytes(cols) || !aligned(ws_dev, 256))
    return GPTQ_EWORKSPACE;
  return run_prepare_hinv(S_H_dev, R_dev, cols, n_total, damp_rel, route, ws_dev, info_dev,
                          static_cast<cudaStream_t>(stream));
}

gptq_status gptq_quantize_layer(const void* W_dev, gptq_dtype w_dtype, int64_t rows, int64_t cols,
                                int64_t ldw, const float* R_dev, int bits, int group, int block,
                                float* W_hat_dev, uint8_t* codes_dev, float* scales_dev,
                                uint8_t* zeros_dev, float* err_sq_dev, void* ws_dev,
                                size_t ws_bytes, int32_t* info_dev, void* stream) {
  const gptq_status st = check_quantize_args(W_dev, w_dtype, rows, cols, ldw, R_dev, bits, group,
                                             block, W_hat_dev, codes_dev, scales_dev, zeros_dev);
  if (st != GPTQ_OK) return st;
  if (ws_dev == nullptr || ws_bytes < quantize_workspace_bytes(rows, cols, block) ||
      !aligned(ws_dev, 256))
    return GPTQ_EWORKSPACE;
  return run_quantize_layer(W_dev, w_dtype, rows, cols, ldw, R_dev, bits, group, block, W_hat_dev,
                            codes_dev, scales_dev, zeros_dev, err_sq_dev, ws_dev, info_dev,
                            static_cast<cudaStream_t>(stream));
}

gptq_status gptq_pack_codes_4bit(const uint8_t* codes_dev, int64_t rows, int64_t cols, int64_t ldc,
                                 uint32_t* packed_dev, int32_t* info_dev, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || ldc < cols || ldc % 8 != 0) return GPTQ_EINVAL;
  if (rows == 0) return GPTQ_OK;  // empty: the buffers may be absent
  if (codes_dev == nullptr || packed_dev == nullptr) return GPTQ_EINVAL;
  if (!aligned(codes_dev, 8) || !aligned(packed_dev, 4)) return GPTQ_EINVAL;
  return run_pack_codes_4bit(codes_dev, rows, cols, ldc, packed_dev, info_dev,
                             static_cast<cudaStream_t>(stream));
}

gptq_status gptq_pack_codes_3bit(const uint8_t* codes_dev, int64_t rows, int64_t cols, int64_t ldc,
                                 uint32_t* packed_dev, int32_t* info_dev, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || ldc < cols || ldc % 8 != 0) return GPTQ_EINVAL;
  if (rows == 0) return GPTQ_OK;  // empty: the buffers may be absent
  if (codes_dev == nullptr || packed_dev == nullptr) return GPTQ_EINVAL;
  if (!aligned(codes_dev, 8) || !aligned(packed_dev, 4)) return GPTQ_EINVAL;
  return run_pack_codes_3bit(codes_dev, rows, cols, ldc, packed_dev, info_dev,
                             static_cast<cudaStream_t>(stream));
}

gptq_status gptq_w4a16_matmul(const uint32_t* packed_dev, const float* scales_dev,
                              const uint8_t* zeros_dev, int64_t rows, int64_t cols, int group,
                              const void* X_dev, gptq_dtype x_dtype, int64_t n, int64_t ldx,
                              float* Y_dev, int64_t ldy, int32_t* info_dev, void* stream) {
  if (rows < 0 || n < 0 || cols <= 0 || cols % 32 != 0) return GPTQ_EINVAL;
  if (group != -1 && (group <= 0 || group % 128 != 0 || cols % group != 0)) return GPTQ_EINVAL;
  if (ldx < cols || ldx % 8 != 0 || ldy < rows) return GPTQ_EINVAL;
  if (x_dtype != GPTQ_BF16) return x_dtype == GPTQ_FP32 ? GPTQ_EUNSUPPORTED : GPTQ_EINVAL;
  if (n > (static_cast<int64_t>(65535) * 128)) return GPTQ_EUNSUPPORTED;
  if (rows > (static_cast<int64_t>(1) << 27) || cols > (static_cast<int64_t>(1) << 22) ||
      rows * (group > 0 ? cols / group : 1) >= (static_cast<int64_t>(1) << 31))
    return GPTQ_EUNSUPPORTED;
  if (rows == 0 || n == 0) return GPTQ_OK;  // empty: the buffers may be absent
  if (packed_dev == nullptr || scales_dev == nullptr || zeros_dev == nullptr || X_dev == nullptr ||
      Y_dev == nullptr)
    return GPTQ_EINVAL;
  if (!aligned(packed_dev, 16) || !aligned(X_dev, 16)) return GPTQ_EINVAL;
  if (n > 16)
    return run_w4a16_gemm(packed_dev, scales_dev, zeros_dev, rows, cols, group, X_dev, n, ldx,
                          Y_dev, ldy, info_dev, static_cast<cudaStream_t>(stream));
  return run_w4a16_gemv(packed_dev, scales_dev, zeros_dev, rows, cols, group, X_dev, n, ldx, Y_dev,
                        ldy, info_dev, static_cast<cudaStream_t>(stream));
}

int gptq_hadamard_block(int64_t n) { return hadamard_block_order(n); }

gptq_status gptq_hadamard_rotate(const void* X_dev, gptq_dtype x_dtype, int64_t rows, int64_t n,
                                 int64_t ldx, const uint32_t* sign_bits_dev, void* Y_dev,
                                 gptq_dtype y_dtype, int64_t ldy, void* stream) {
  if (rows < 0 || n <= 0 || n % 32 != 0 || ldx < n || ldy < n) return GPTQ_EINVAL;
  if ((x_dtype != GPTQ_BF16 && x_dtype != GPTQ_FP32) ||
      (y_dtype != GPTQ_BF16 && y_dtype != GPTQ_FP32))
    return GPTQ_EINVAL;
  const int64_t xe = x_dtype == GPTQ_BF16 ? 2 : 4, ye = y_dtype == GPTQ_BF16 ? 2 : 4;
  if ((ldx * xe) % 16 != 0 || (ldy * ye) % 16 != 0) return GPTQ_EINVAL;
  if (rows == 0) return GPTQ_OK;  // empty: the buffers may be absent
  if (X_dev == nullptr || Y_dev == nullptr) return GPTQ_EINVAL;
  if (!aligned(X_dev, 16) || !aligned(Y_dev, 16) || !aligned(sign_bits_dev, 4)) return GPTQ_EINVAL;
  if (X_dev == Y_dev && (x_dtype != y_dtype || ldx != ldy)) return GPTQ_EINVAL;
  return run_hadamard_rotate(X_dev, x_dtype == GPTQ_BF16, ldx, rows, n, sign_bits_dev, Y_dev,
                             y_dtype == GPTQ_BF16, ldy, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_obq_quantize(const float* W_dev, int64_t rows, int64_t cols, int64_t ldw,
                              const double* Hinv_dev, int bits, int order_mode,
                              uint8_t* codes_dev, float* W_hat_dev, int32_t* order_dev,
                              double* loss_dev, float* scales_dev, uint8_t* zeros_dev,
                              void* stream) {
  if (rows < 0 || cols < 1 || ldw < cols || bits < 2 || bits > 8) return GPTQ_EINVAL;
  if (order_mode != GPTQ_OBQ_NATURAL && order_mode != GPTQ_OBQ_GREEDY) return GPTQ_EINVAL;
  if (cols > 128) return GPTQ_EUNSUPPORTED;
  if (rows == 0) return GPTQ_OK;  // empty: the buffers may be absent
  if (W_dev == nullptr || Hinv_dev == nullptr || codes_dev == nullptr || W_hat_dev == nullptr)
    return GPTQ_EINVAL;
  return run_obq_quantize(W_dev, rows, cols, ldw, Hinv_dev, bits, order_mode == GPTQ_OBQ_GREEDY,
                          codes_dev, W_hat_dev, order_dev, loss_dev, scales_dev, zeros_dev,
                          static_cast<cudaStream_t>(stream));
}

size_t gptq_workspace_size(int which, int64_t rows, int64_t cols, int block) {
  if (cols <= 0) return 0;
  if (which == GPTQ_WS_PREPARE) return prepare_workspace_bytes(cols);
  if (which == GPTQ_WS_QUANTIZE) {
    if (rows <= 0 || (block != 32 && block != 64 && block != 128)) return 0;
    return quantize_workspace_bytes(rows, cols, block);
  }
  return 0;
}

gptq_status gptq_info_status(int32_t info) {
  if (info == GPTQ_INFO_OK) return GPTQ_OK;
  if (info > 0) return GPTQ_ENOTPD;
  if (info == GPTQ_INFO_TIMEOUT) return GPTQ_ETIMEOUT;
  return GPTQ_EINVAL;
}

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "GPTQ_OK";
    case GPTQ_EINVAL: return "GPTQ_EINVAL: invalid argument";
    case GPTQ_ENOTPD: return "GPTQ_ENOTPD: matrix not positive definite";
    case GPTQ_ECUDA: return "GPTQ_ECUDA: CUDA runtime error";
    case GPTQ_EUNSUPPORTED: return "GPTQ_EUNSUPPORTED: unsupported size or type";
    case GPTQ_ETIMEOUT: return "GPTQ_ETIMEOUT: bounded device wait expired";
    case GPTQ_EWORKSPACE: return "GPTQ_EWORKSPACE: workspace missing or too small";
    default: return "unknown gptq_status";
  }
}

uint64_t gptq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

gptq_status gptq_selftest_wait_timeout(int32_t* info_dev, int limit_ms, void* stream) {
  if (info_dev == nullptr || limit_ms < 1 || limit_ms > 10000) return GPTQ_EINVAL;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      info_dev, static_cast<uint64_t>(limit_ms) * 1000000ull);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

gptq_status gptq_selftest_flag_timeout(const int32_t* flag_dev, int32_t* info_dev, int limit_ms,
                                       void* stream) {
  if (flag_dev == nullptr || info_dev == nullptr || limit_ms < 1 || limit_ms > 10000)
    return GPTQ_EINVAL;
  if (!aligned(flag_dev, 4)) return GPTQ_EINVAL;
  selftest_flag_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      flag_dev, info_dev, static_cast<uint64_t>(limit_ms) * 1000000ull);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

gptq_status gptq_selftest_gemm(const float* A_dev, int64_t lda, int a_mn, const float* B_dev,
                               int64_t ldb, int b_mn, float* C_dev, int64_t ldc, int M, int N,
                               int K, float alpha, float beta, int lower, int klo_from_m,
                               int klo_from_n, float* C_big_dev, float* C_small_dev, void* ws_dev,
                               size_t ws_bytes, int32_t* info_dev, void* stream) {
  if (A_dev == nullptr || B_dev == nullptr || ws_dev == nullptr || M <= 0 || N <= 0 || K < 0)
    return GPTQ_EINVAL;
  if (lda % 4 || ldb % 4 || ldc % 4 || (C_big_dev != nullptr) != (C_small_dev != nullptr))
    return GPTQ_EINVAL;
  if ((C_dev == nullptr && beta != 0.f) || !aligned(ws_dev, 256)) return GPTQ_EINVAL;
  const int64_t ra = a_mn ? K : M, ca = a_mn ? M : K;
  const int64_t rb = b_mn ? K : N, cb = b_mn ? N : K;
  if (lda < ca || ldb < cb || (C_dev != nullptr && ldc < N)) return GPTQ_EINVAL;
  const size_t a_bytes = align_up(static_cast<size_t>(ra) * lda * 4, 256);
  const size_t b_bytes = align_up(static_cast<size_t>(rb) * ldb * 4, 256);
  if (ws_bytes < 2 * a_bytes + 2 * b_bytes) return GPTQ_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws_dev);
  float* Ab = reinterpret_cast<float*>(w);
  float* As = reinterpret_cast<float*>(w + a_bytes);
  float* Bb = reinterpret_cast<float*>(w + 2 * a_bytes);
  float* Bs = reinterpret_cast<float*>(w + 2 * a_bytes + b_bytes);
  gptq_status st = launch_split_tf32(A_dev, lda, ra, ca, Ab, As, lda, s);
  if (st != GPTQ_OK) return st;
  if ((st = launch_split_tf32(B_dev, ldb, rb, cb, Bb, Bs, ldb, s)) != GPTQ_OK) return st;
  TcGemmArgs g{Ab, As, Bb, Bs, lda, ldb, a_mn ? 1 : 0, b_mn ? 1 : 0, M, N, K, alpha, beta,
               lower ? 1 : 0, klo_from_m ? 1 : 0, klo_from_n ? 1 : 0, C_dev, ldc, C_big_dev,
               C_small_dev, ldc, info_dev};
  return launch_gemm_tc(g, s);
}

const char* gptq_version(void) { return "0.1.0"; }

}  // extern "C"
