// OBQ: greedy-order quantization with explicit inverse-Hessian downdates, the reference GPTQ's
// fixed column order is measured against (small layers, at most 128 columns).
//
// "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)":
//   "Greedy Search"          each step quantizes the remaining weight whose quantization raises
//                            the proxy loss least: (w_p - q_p)^2 / H^-1[p, p] (up to a factor 2);
//   "Generalized Weight Update"  the other weights move by -(w_p - q_p) H^-1[:, p] / H^-1[p, p];
//   "The OBS / GPTQ Trick"   H^-1 of the remaining weights = H^-1 - H^-1[:, p] H^-1[p, :] / H^-1[p, p];
//   "Limitations of OBQ"     every row needs its own copy of H^-1.
//
// One CTA per row. Its copy of H^-1 (fp64) lives in registers: thread t holds row t mod 128,
// columns 64 * (t / 128) .. + 63. Each step: the remaining columns are scored in parallel and the
// minimum found (ties to the lowest column); the pivot row of H^-1 (equal to its column: H^-1 is
// symmetric) is published through shared memory; the weights, the diagonal and every register
// entry are downdated. All fp64 and fp32 operations are the intrinsic round-to-nearest forms, in
// the order the arithmetic is written, with no fused multiply-adds, so the result is reproducible
// operation by operation.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace gptq {
namespace {

constexpr int kMaxCols = 128;
constexpr int kThreads = 256;
constexpr int kHalf = 64;  // H^-1 columns a thread keeps in registers

__global__ void __launch_bounds__(kThreads, 1)
obq_rows_kernel(const float* __restrict__ W, int64_t ldw, int cols,
                const double* __restrict__ Hinv, int bits, int greedy, uint8_t* __restrict__ codes,
                float* __restrict__ W_hat, int32_t* __restrict__ order, double* __restrict__ loss,
                float* __restrict__ scales, uint8_t* __restrict__ zeros) {
  __shared__ double w[kMaxCols], diag[kMaxCols], h[kMaxCols], g[kMaxCols], dv[kMaxCols];
  __shared__ float whv[kMaxCols], qv[kMaxCols];
  __shared__ int removed[kMaxCols];
  __shared__ double red_s[kMaxCols / 32];
  __shared__ int red_i[kMaxCols / 32];
  __shared__ float red_lo[kThreads / 32], red_hi[kThreads / 32];
  __shared__ float grid_s, grid_z;
  __shared__ int piv;
  __shared__ double e_sh;
  griddep_wait();

  const double kInf = __longlong_as_double(0x7FF0000000000000LL);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int i = t & (kMaxCols - 1), half = t / kMaxCols;
  const int64_t row = blockIdx.x;
  const float* wr = W + row * ldw;
  const float maxq = static_cast<float>((1 << bits) - 1);

  double R[kHalf];
#pragma unroll
  for (int k = 0; k < kHalf; ++k) {
    const int col = kHalf * half + k;
    R[k] = (i < cols && col < cols) ? Hinv[static_cast<int64_t>(i) * cols + col] : 0.0;
  }
  if (t < kMaxCols) {
    w[t] = t < cols ? static_cast<double>(wr[t]) : 0.0;
    diag[t] = t < cols ? Hinv[static_cast<int64_t>(t) * cols + t] : 1.0;
    removed[t] = t >= cols;
  }

  // Per-row grid in float32 from the original row: lo = min(0, min w), hi = max(0, max w);
  // an all-zero row uses [-1, 1]; s = (hi - lo) / (2^k - 1), z = clamp(rint(-lo / s), 0, 2^k - 1).
  float lo = 0.f, hi = 0.f;
  for (int j = t; j < cols; j += kThreads) {
    const float v = wr[j];
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if (lane == 0) {
    red_lo[warp] = lo;
    red_hi[warp] = hi;
  }
  __syncthreads();
  if (t == 0) {
    for (int k = 1; k < kThreads / 32; ++k) {
      lo = fminf(lo, red_lo[k]);
      hi = fmaxf(hi, red_hi[k]);
    }
    if (lo == hi) {
      lo = -1.f;
      hi = 1.f;
    }
    const float s = __fdiv_rn(__fsub_rn(hi, lo), maxq);
    grid_s = s;
    grid_z = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), maxq);
  }
  __syncthreads();
  const float s = grid_s, z = grid_z;

  double loss_acc = 0.0;  // thread 0's running sum
  for (int step = 0; step < cols; ++step) {
    // score every remaining column: the float32 grid decision, then d^2 / H^-1[j, j] in fp64
    if (t < kMaxCols) {
      const int j = t;
      double score = kInf;
      if (!removed[j]) {
        const float w32 = __double2float_rn(w[j]);
        const float qf = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w32, s)), z), 0.f), maxq);
        const float wh = __fmul_rn(s, __fsub_rn(qf, z));
        const double d = __dsub_rn(w[j], static_cast<double>(wh));
        dv[j] = d;
        whv[j] = wh;
        qv[j] = qf;
        score = greedy ? __ddiv_rn(__dmul_rn(d, d), diag[j]) : (j == step ? 0.0 : kInf);
      }
      int jbest = j;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const double os = __shfl_xor_sync(0xffffffffu, score, off);
        const int oj = __shfl_xor_sync(0xffffffffu, jbest, off);
        if (os < score || (os == score && oj < jbest)) {
          score = os;
          jbest = oj;
        }
      }
      if (lane == 0) {
        red_s[warp] = score;
        red_i[warp] = jbest;
      }
    }
    __syncthreads();
    if (t == 0) {
      double best = red_s[0];
      int p = red_i[0];
      for (int k = 1; k < kMaxCols / 32; ++k)
        if (red_s[k] < best || (red_s[k] == best && red_i[k] < p)) {
          best = red_s[k];
          p = red_i[k];
        }
      piv = p;
      const double dp = dv[p];
      loss_acc = __dadd_rn(loss_acc, __ddiv_rn(__dmul_rn(dp, dp), diag[p]));
      e_sh = __ddiv_rn(dp, diag[p]);
      removed[p] = 1;
      codes[row * cols + p] = static_cast<uint8_t>(qv[p]);
      W_hat[row * cols + p] = whv[p];
      if (order != nullptr) order[row * cols + step] = p;
    }
    __syncthreads();
    const int p = piv;
    if (i == p) {  // publish row p of H^-1 (two threads, one per column half)
#pragma unroll
      for (int k = 0; k < kHalf; ++k) h[kHalf * half + k] = R[k];
    }
    __syncthreads();
    if (t < kMaxCols) {
      const int j = t;
      const double gj = __ddiv_rn(h[j], h[p]);
      g[j] = gj;
      w[j] = __dsub_rn(w[j], __dmul_rn(e_sh, h[j]));  // compensation of the other weights
      diag[j] = __dsub_rn(diag[j], __dmul_rn(h[j], gj));
    }
    __syncthreads();
    const double hi_row = h[i];
#pragma unroll
    for (int k = 0; k < kHalf; ++k) R[k] = __dsub_rn(R[k], __dmul_rn(hi_row, g[kHalf * half + k]));
  }
  griddep_launch_dependents();
  if (t == 0) {
    if (loss != nullptr) loss[row] = loss_acc;
    if (scales != nullptr) scales[row] = s;
    if (zeros != nullptr) zeros[row] = static_cast<uint8_t>(z);
  }
}

}  // namespace

gptq_status run_obq_quantize(const float* W, int64_t rows, int64_t cols, int64_t ldw,
                             const double* Hinv, int bits, int greedy, uint8_t* codes,
                             float* W_hat, int32_t* order, double* loss, float* scales,
                             uint8_t* zeros, cudaStream_t stream) {
  if (rows > 0x7FFFFFFF) return GPTQ_EUNSUPPORTED;
  return launch_pdl(obq_rows_kernel, dim3(static_cast<unsigned>(rows)), dim3(kThreads), 0, stream,
                    W, ldw, static_cast<int>(cols), Hinv, bits, greedy, codes, W_hat, order, loss,
                    scales, zeros);
}

}  // namespace gptq
