// gptq_quantize_layer_noalloc: the column loop for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: their host framework owns every
// device allocation through its own pool (a direct cudaMalloc there fails or breaks the pool's
// accounting), or they run in a loop where cudaMalloc's implicit device-wide synchronization is
// not acceptable. This entry point needs no workspace: the error buffer E lives in a fixed-size
// array compiled into this library. The caller still passes every input and output buffer.
//
// The array is a file-scope __device__ variable, so every GPU that loads the library holds
// GPTQ_NOALLOC_SCRATCH_BYTES of it until the process exits. Host code may not use the array's
// name as a device pointer (on the host it is only a stand-in symbol); its device address is
// looked up once per device with cudaGetSymbolAddress, with that device current, and cached for
// the life of the process. A cudaDeviceReset destroys the context that holds the array, so the
// cached address is stale afterwards: this entry point must not be used on a device after it has
// been reset.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace gptq {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GPTQ_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_dev[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up on first use).
gptq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPTQ_ECUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return GPTQ_ECUDA;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return GPTQ_OK;
}
}  // namespace

}  // namespace gptq

extern "C" gptq_status gptq_quantize_layer_noalloc(
    const void* W_dev, gptq_dtype w_dtype, int64_t rows, int64_t cols, int64_t ldw,
    const float* R_dev, int bits, int group, int block, float* W_hat_dev, uint8_t* codes_dev,
    float* scales_dev, uint8_t* zeros_dev, float* err_sq_dev, int32_t* info_dev, void* stream) {
  using namespace gptq;
  // The ordinary argument checks come first, so a call that gptq_quantize_layer would refuse for
  // its arguments is refused here for the same reason; only a valid call that is too large for
  // the built-in scratch gets GPTQ_EWORKSPACE.
  const gptq_status bad = check_quantize_args(W_dev, w_dtype, rows, cols, ldw, R_dev, bits, group,
                                              block, W_hat_dev, codes_dev, scales_dev, zeros_dev);
  if (bad != GPTQ_OK) return bad;
  const size_t need = quantize_workspace_bytes(rows, cols, block);
  if (need > GPTQ_NOALLOC_SCRATCH_BYTES) return GPTQ_EWORKSPACE;
  void* scratch = nullptr;
  const gptq_status st = scratch_address(&scratch);
  if (st != GPTQ_OK) return st;
  // Same validation and kernels as gptq_quantize_layer, with the built-in scratch as workspace.
  return gptq_quantize_layer(W_dev, w_dtype, rows, cols, ldw, R_dev, bits, group, block, W_hat_dev,
                             codes_dev, scales_dev, zeros_dev, err_sq_dev, scratch,
                             GPTQ_NOALLOC_SCRATCH_BYTES, info_dev, stream);
}
