// Data-free randomized Hadamard rotation of the input-channel axis, applied before GPTQ.
//
// "OptRot: Mitigating Weight Outliers via Data-Free Rotations for Post-Training Quantization",
// Abstract and Figure 1: a rotation fused into the weights (W Q) and, transposed, into the
// activations (X Q for token-major X) leaves the layer output unchanged while spreading weight
// outliers; Theorem 3.1 bounds the round-to-nearest error by the weight incoherence, which the
// rotation lowers. Q = diag(signs) (I (x) H_b) / sqrt(b) with the Sylvester Hadamard matrix H_b,
// b = the largest power of two dividing n, at most 4096.
//
// One CTA rotates 4096 consecutive elements of segments (a segment = b contiguous columns of one
// row): 128 threads x 32 values in registers. The transform of order 2^L runs as butterfly
// passes of up to five index bits each inside a thread's registers, with the segment transposed
// through shared memory between passes so the next five bits become register bits. HBM-bound:
// every element is read once and written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace gptq {
namespace {

constexpr int kTile = 4096;      // elements per CTA
constexpr int kThreads = 128;    // 32 elements per thread

// Shared-memory index with one pad word per 32, so the transposed accesses below spread over
// the banks.
__device__ __forceinline__ int pad(int e) { return e + (e >> 5); }

// Unnormalised butterflies over register-index bits 0 .. M-1 of v (groups of 2^M registers).
template <int M>
__device__ __forceinline__ void butterflies(float (&v)[32]) {
#pragma unroll
  for (int h = 1; h < (1 << M); h <<= 1)
#pragma unroll
    for (int k = 0; k < 32; ++k)
      if ((k & h) == 0) {
        const float a = v[k], c = v[k + h];
        v[k] = a + c;
        v[k + h] = a - c;
      }
}

// Pass over segment index bits LO .. LO+M-1: a thread holds, in register k = jb + (ja << M),
// element e = low(r) | jb << LO | high(r) << (LO + M) with r = ja + (u << (5 - M)), where low()
// keeps r's bits below LO. Over the segment's threads u this visits every element once.
template <int LO, int M>
__device__ __forceinline__ int pass_index(int u, int k) {
  const int jb = k & ((1 << M) - 1), ja = k >> M;
  const int r = ja + (u << (5 - M));
  return (r & ((1 << LO) - 1)) | (jb << LO) | ((r >> LO) << (LO + M));
}

template <int LO, int M>
__device__ __forceinline__ void smem_pass(float (&v)[32], float* sm, int base, int u) {
#pragma unroll
  for (int k = 0; k < 32; ++k) v[k] = sm[pad(base + pass_index<LO, M>(u, k))];
  butterflies<M>(v);
  // Each element of the segment is read and written by the same thread in this pass.
#pragma unroll
  for (int k = 0; k < 32; ++k) sm[pad(base + pass_index<LO, M>(u, k))] = v[k];
}

// Y[row, blk*b + i] = sum_j X[row, blk*b + j] * s_j * H_b[j][i] / sqrt(b), b = 2^L.
template <int L>
__global__ void __launch_bounds__(kThreads)
hadamard_rotate_kernel(const void* __restrict__ X, int x_bf16, int64_t ldx, int64_t rows,
                       int64_t n, const uint32_t* __restrict__ sign_bits, void* Y, int y_bf16,
                       int64_t ldy, float scale) {
  constexpr int B = 1 << L;           // Hadamard block order
  constexpr int TPS = B / 32;         // threads per segment
  constexpr int SPT = kTile / B;      // segments per CTA
  __shared__ float sm[kTile + kTile / 32];
  griddep_wait();

  const int t = threadIdx.x;
  const int s_local = t / TPS, u = t % TPS;
  const int64_t nblk = n / B;
  const int64_t seg = static_cast<int64_t>(blockIdx.x) * SPT + s_local;
  const bool live = seg < rows * nblk;
  const int64_t row = live ? seg / nblk : 0, blk = live ? seg - row * nblk : 0;
  const int64_t col0 = blk * B + 32 * u;  // this thread's first column

  float v[32];
  if (live) {
    if (x_bf16) {
      const uint4* p = reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(X) + row * ldx + col0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 q = __ldg(p + i);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
          v[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
      }
    } else {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(X) + row * ldx +
                                                        col0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 q = __ldg(p + i);
        v[4 * i] = q.x;
        v[4 * i + 1] = q.y;
        v[4 * i + 2] = q.z;
        v[4 * i + 3] = q.w;
      }
    }
    if (sign_bits != nullptr) {
      const uint32_t m = __ldg(sign_bits + col0 / 32);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((m >> j) & 1u) << 31));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = 0.f;
  }

  butterflies<5>(v);  // index bits 0..4: a thread's own 32 consecutive elements
  if constexpr (L > 5) {
    const int base = s_local * B;
#pragma unroll
    for (int j = 0; j < 32; ++j) sm[pad(base + 32 * u + j)] = v[j];
    __syncthreads();
    smem_pass<5, (L - 5 < 5 ? L - 5 : 5)>(v, sm, base, u);  // bits 5..9
    if constexpr (L > 10) {
      __syncthreads();
      smem_pass<10, L - 10>(v, sm, base, u);  // bits 10..11
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = sm[pad(base + 32 * u + j)];
  }
  griddep_launch_dependents();
  if (!live) return;

  if (y_bf16) {
    uint4* p = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(Y) + row * ldy + col0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h =
            __floats2bfloat162_rn(v[8 * i + 2 * e] * scale, v[8 * i + 2 * e + 1] * scale);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      p[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(Y) + row * ldy + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      p[i] = make_float4(v[4 * i] * scale, v[4 * i + 1] * scale, v[4 * i + 2] * scale,
                         v[4 * i + 3] * scale);
  }
}

template <int L>
gptq_status launch_rotate(const void* X, int x_bf16, int64_t ldx, int64_t rows, int64_t n,
                          const uint32_t* sign_bits, void* Y, int y_bf16, int64_t ldy,
                          cudaStream_t stream) {
  constexpr int B = 1 << L;
  const int64_t segs = rows * (n / B);
  const int64_t ctas = (segs + kTile / B - 1) / (kTile / B);
  if (ctas > 0x7FFFFFFF) return GPTQ_EUNSUPPORTED;
  // 1 / sqrt(2^L): a power of two for even L (exact), else rounded once in float.
  const float scale = (L % 2 == 0) ? 1.0f / static_cast<float>(1 << (L / 2))
                                   : 1.0f / sqrtf(static_cast<float>(B));
  return launch_pdl(hadamard_rotate_kernel<L>, dim3(static_cast<unsigned>(ctas)), dim3(kThreads),
                    0, stream, X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, scale);
}

}  // namespace

int hadamard_block_order(int64_t n) {
  if (n <= 0) return 0;
  int64_t b = n & -n;
  if (b > kTile) b = kTile;
  return static_cast<int>(b);
}

gptq_status run_hadamard_rotate(const void* X, int x_bf16, int64_t ldx, int64_t rows, int64_t n,
                                const uint32_t* sign_bits, void* Y, int y_bf16, int64_t ldy,
                                cudaStream_t stream) {
  switch (hadamard_block_order(n)) {
    case 32: return launch_rotate<5>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 64: return launch_rotate<6>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 128: return launch_rotate<7>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 256: return launch_rotate<8>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 512: return launch_rotate<9>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 1024:
      return launch_rotate<10>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 2048:
      return launch_rotate<11>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    case 4096:
      return launch_rotate<12>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    default: return GPTQ_EINVAL;
  }
}

}  // namespace gptq
