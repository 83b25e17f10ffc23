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
#include <algorithm>

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

// ---------------------------------------------------------------------------------------------
// Block order 4096, the order of every width that is a multiple of 4096. One CTA of 64 threads
// owns one 4096-element segment at a time and loops over segments (a persistent grid). Each
// thread holds 64 values, so the 12 index bits e0..e11 take two register passes:
//   pass A: a thread u holds e0..e2 and e9..e11 (registers), u = e3..e8. Its values arrive as
//           eight 16-byte runs of 8 consecutive elements, 512 apart: coalesced global loads.
//   pass B: a thread holds e3..e8 (registers), its index gives e0..e2 and e9..e11.
// The segment goes through one shared buffer between the passes and back into the pass-A layout
// for the coalesced store. The butterflies run as packed f32x2 adds (round to nearest, like the
// scalar add), two lanes per instruction; the one stage inside a pair stays scalar.
namespace h12 {
constexpr int kThreads = 64;
// Shared layout: the 8-element run (j, u) = elements 512 j + 8 u .. +7 starts at word
// j * kRowPitch + 8 u + 4 (u / 4). Pass A's 16-byte accesses (8 lanes u = 8w .. 8w+7 per phase)
// land in 8 distinct 16-byte bank groups, and pass B's 32-bit accesses (lanes over e0..e2, e9,
// e10) in 32 distinct banks, since kRowPitch = 8 (mod 32) with an odd quotient.
constexpr int kRowPitch = 584;
constexpr int kBufWords = 8 * kRowPitch;
constexpr int kMaxSignWords = 2048;   // widths up to 65536 keep their signs in shared memory
constexpr int kMaxCtasPerSm = 8;

__device__ __forceinline__ int run_word(int j, int u) { return j * kRowPitch + 8 * u + 4 * (u >> 2); }
}  // namespace h12

// (a0, a1), (c0, c1) <- (a0 + c0, a1 + c1), (a0 - c0, a1 - c1) as two packed f32x2 operations.
__device__ __forceinline__ void butterfly_x2(float& a0, float& a1, float& c0, float& c1) {
  asm("{\n\t.reg .b64 a, c, s, d;\n\t"
      "mov.b64 a, {%0, %1};\n\tmov.b64 c, {%2, %3};\n\t"
      "add.rn.f32x2 s, a, c;\n\tsub.rn.f32x2 d, a, c;\n\t"
      "mov.b64 {%0, %1}, s;\n\tmov.b64 {%2, %3}, d;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(c0), "+f"(c1));
}

// Unnormalised transform over all six register-index bits of v: bits 1..5 on (v[2p], v[2p+1])
// pairs, then bit 0 inside each pair.
__device__ __forceinline__ void butterflies64(float (&v)[64]) {
#pragma unroll
  for (int h = 2; h < 64; h <<= 1)
#pragma unroll
    for (int k = 0; k < 64; k += 2)
      if ((k & h) == 0) butterfly_x2(v[k], v[k + 1], v[k + h], v[k + h + 1]);
#pragma unroll
  for (int k = 0; k < 64; k += 2) {
    const float a = v[k], c = v[k + 1];
    v[k] = a + c;
    v[k + 1] = a - c;
  }
}

// bf16 sign words are stored with the signs of even columns in bits 0..15 and of odd columns in
// bits 16..31, so one shift lines up the two signs of a bf16 pair with bits 15 and 31.
__device__ __forceinline__ uint32_t split_even_odd(uint32_t w) {
  uint32_t p = 0;
  for (int b = 0; b < 16; ++b)
    p |= (((w >> (2 * b)) & 1u) << b) | (((w >> (2 * b + 1)) & 1u) << (16 + b));
  return p;
}

template <bool XB, bool YB>
__global__ void __launch_bounds__(h12::kThreads, h12::kMaxCtasPerSm)
hadamard4096_kernel(const void* __restrict__ X, int64_t ldx, uint32_t segs, uint32_t nblk,
                    const uint32_t* __restrict__ sign_bits, int sign_words, void* Y, int64_t ldy) {
  using namespace h12;
  extern __shared__ __align__(16) float sh[];
  float* buf = sh;
  uint32_t* sgn = reinterpret_cast<uint32_t*>(sh + kBufWords);
  const int u = threadIdx.x;
  const int q = u & 3;              // which byte of a 32-column sign word holds this run

  griddep_wait();
  for (int i = u; i < sign_words; i += h12::kThreads) {
    const uint32_t w = sign_bits != nullptr ? __ldg(sign_bits + i) : 0u;
    sgn[i] = XB ? split_even_odd(w) : w;
  }
  __syncthreads();

  uint32_t g = blockIdx.x;
  if (g >= segs) return;  // uniform over the CTA

  // pass-A raw loads: run j of segment g is 16 bytes (bf16) at column 512 j + 8 u
  uint4 raw[XB ? 8 : 1];
  auto seg_base = [&](uint32_t gg, int64_t ld, int64_t& row, uint32_t& blk) {
    row = static_cast<int64_t>(gg / nblk);
    blk = gg - static_cast<uint32_t>(row) * nblk;
    return row * ld + static_cast<int64_t>(blk) * 4096 + 8 * u;
  };
  if constexpr (XB) {
    int64_t row;
    uint32_t blk;
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(X) +
                                                    seg_base(g, ldx, row, blk));
#pragma unroll
    for (int j = 0; j < 8; ++j) raw[j] = __ldg(p + 64 * j);
  }

  for (;;) {
    int64_t row;
    uint32_t blk;
    const int64_t xoff = seg_base(g, ldx, row, blk);
    const uint32_t* sg = sgn + blk * 128 + (u >> 2);  // + 16 j: run j's sign word
    float v[64];
    if constexpr (XB) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t P = sg[16 * j];
        const uint32_t w4[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          // bits 15 and 31 of P << (15 - 4q - m) are the signs of columns 8q + 2m and 8q + 2m + 1
          const uint32_t w = w4[m] ^ ((P << (15 - 4 * q - m)) & 0x80008000u);
          v[8 * j + 2 * m] = __uint_as_float(w << 16);
          v[8 * j + 2 * m + 1] = __uint_as_float(w & 0xFFFF0000u);
        }
      }
      const uint32_t next = g + gridDim.x;
      if (next < segs) {  // the next segment's loads fly while this one is transformed
        int64_t row2;
        uint32_t blk2;
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(X) +
                                                        seg_base(next, ldx, row2, blk2));
#pragma unroll
        for (int j = 0; j < 8; ++j) raw[j] = __ldg(p + 64 * j);
      }
    } else {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(X) + xoff);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w = sg[16 * j];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float4 f = __ldg(p + 128 * j + h);
          const float f4[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = 4 * h + i;  // bit 31 of w << (31 - 8q - c) is column 8q + c's sign
            v[8 * j + c] = __uint_as_float(__float_as_uint(f4[i]) ^
                                           ((w << (31 - 8 * q - c)) & 0x80000000u));
          }
        }
      }
    }

    butterflies64(v);  // e0..e2, e9..e11
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4* d = reinterpret_cast<float4*>(buf + run_word(j, u));
      d[0] = make_float4(v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3]);
      d[1] = make_float4(v[8 * j + 4], v[8 * j + 5], v[8 * j + 6], v[8 * j + 7]);
    }
    __syncthreads();
    // pass B: this thread's element e = c0 + 8 k + 512 h sits at run_word(h, k) + c0
    float* bb = buf + (u >> 3) * kRowPitch + (u & 7);
#pragma unroll
    for (int k = 0; k < 64; ++k) v[k] = bb[8 * k + 4 * (k >> 2)];
    butterflies64(v);  // e3..e8
#pragma unroll
    for (int k = 0; k < 64; ++k) bb[8 * k + 4 * (k >> 2)] = v[k];
    __syncthreads();

    const uint32_t next = g + gridDim.x;
    if (next >= segs) griddep_launch_dependents();
    const int64_t yoff = row * ldy + static_cast<int64_t>(blk) * 4096 + 8 * u;
    constexpr float kScale = 1.0f / 64.0f;  // 1 / sqrt(4096), exact
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4* s4 = reinterpret_cast<const float4*>(buf + run_word(j, u));
      const float4 a = s4[0], b = s4[1];
      if constexpr (YB) {
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x * kScale, a.y * kScale);
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(a.z * kScale, a.w * kScale);
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(b.x * kScale, b.y * kScale);
        const __nv_bfloat162 h3 = __floats2bfloat162_rn(b.z * kScale, b.w * kScale);
        uint4 o;
        o.x = *reinterpret_cast<const uint32_t*>(&h0);
        o.y = *reinterpret_cast<const uint32_t*>(&h1);
        o.z = *reinterpret_cast<const uint32_t*>(&h2);
        o.w = *reinterpret_cast<const uint32_t*>(&h3);
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(Y) + yoff)[64 * j] = o;
      } else {
        float4* d = reinterpret_cast<float4*>(static_cast<float*>(Y) + yoff) + 128 * j;
        d[0] = make_float4(a.x * kScale, a.y * kScale, a.z * kScale, a.w * kScale);
        d[1] = make_float4(b.x * kScale, b.y * kScale, b.z * kScale, b.w * kScale);
      }
    }
    if (next >= segs) break;
    g = next;
  }
}

template <bool XB, bool YB>
gptq_status launch_rotate4096(const void* X, int64_t ldx, int64_t rows, int64_t n,
                              const uint32_t* sign_bits, void* Y, int64_t ldy,
                              cudaStream_t stream) {
  using namespace h12;
  const int64_t segs = rows * (n / 4096);
  const int sign_words = static_cast<int>(n / 32);
  const int smem = (kBufWords + sign_words) * 4;
  auto kern = hadamard4096_kernel<XB, YB>;
  gptq_status st = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (st != GPTQ_OK) return st;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, h12::kThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return GPTQ_ECUDA;
  const int64_t grid = std::min<int64_t>(segs, static_cast<int64_t>(per_sm) * num_sms());
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(h12::kThreads),
                    static_cast<size_t>(smem), stream, X, ldx, static_cast<uint32_t>(segs),
                    static_cast<uint32_t>(n / 4096), sign_bits, sign_words, Y, ldy);
}

gptq_status launch_rotate4096_any(const void* X, int x_bf16, int64_t ldx, int64_t rows, int64_t n,
                                  const uint32_t* sign_bits, void* Y, int y_bf16, int64_t ldy,
                                  cudaStream_t stream) {
  if (x_bf16)
    return y_bf16 ? launch_rotate4096<true, true>(X, ldx, rows, n, sign_bits, Y, ldy, stream)
                  : launch_rotate4096<true, false>(X, ldx, rows, n, sign_bits, Y, ldy, stream);
  return y_bf16 ? launch_rotate4096<false, true>(X, ldx, rows, n, sign_bits, Y, ldy, stream)
                : launch_rotate4096<false, false>(X, ldx, rows, n, sign_bits, Y, ldy, stream);
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
      // the two-pass kernel keeps the signs of a row in shared memory and counts segments in
      // 32 bits; wider or taller inputs take the three-pass kernel
      if (n / 32 <= h12::kMaxSignWords && rows * (n / 4096) <= 0x7FFFFFFF)
        return launch_rotate4096_any(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
      return launch_rotate<12>(X, x_bf16, ldx, rows, n, sign_bits, Y, y_bf16, ldy, stream);
    default: return GPTQ_EINVAL;
  }
}

}  // namespace gptq
