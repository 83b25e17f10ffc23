// S2-S5 -- from the accumulated S to the upper factor R of the damped inverse Hessian.
//
// "GPTQ second-order quantization" blog, "The objective is layer output" (H = 2 X X^T) and
// "3. Cholesky reformulation" (damping about 1 % of the mean diagonal; one Cholesky up front);
// "Part 3: Adaptive Rounding: GPTQ", "Observation 3" and "Algorithm GPTQ" (Cholesky of H^-1,
// whose rows are read during quantization).
//
// Two routes to the same R (the upper factor with positive diagonal is unique):
//  * three-step, as the pages write it: H_d = L L^T (blocked right-looking Cholesky, 128-wide
//    panels), L^-1 (blocked triangular inverse, row block by row block), H_d^-1 = L^-T L^-1
//    (triangular product, lower half only), H_d^-1 = L2 L2^T (second Cholesky), R = L2^T;
//  * reversed: with J the order-reversing permutation, J H_d J = M M^T (one Cholesky), so
//    H_d = U U^T with U = J M J upper, H_d^-1 = U^-T U^-1 and R = U^-1 = J M^-1 J: one Cholesky
//    and one triangular inverse, half the flops and half the chain of diagonal blocks.
// Each 128 x 128 diagonal block is factored and inverted on chip by one CTA; everything else is a
// 3xTF32 tensor-core matrix product whose operands are kept as tf32 (big, small) pairs in the
// workspace.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace la {
constexpr int kNB = 128;       // panel / diagonal block width
constexpr int kLd = kNB + 1;   // padded shared-memory row
constexpr int kDiagThreads = 512;
constexpr int kDiagSmem = (2 * kNB * kLd + 3 * 32 * 33) * 4;
}  // namespace la

#define GPTQ_TRY(x)               \
  do {                            \
    gptq_status _s = (x);         \
    if (_s != GPTQ_OK) return _s; \
  } while (0)

__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// ------------------------------------------------------------------------------------------------
// S2: lambda from the diagonal, then H = (2/N) S mirrored, and H_d = H + lambda I into R (lower).
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
diag_lambda_kernel(const float* S, int64_t n, double scale, float damp_rel, float* lam_out,
                   int32_t* info) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += static_cast<double>(S[i * n + i]);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) {
      const double mean_h = scale * s / static_cast<double>(n);
      if (!(mean_h > 0.0) || !isfinite(mean_h)) record_info(info, GPTQ_INFO_BAD_HESSIAN);
      lam_out[0] = static_cast<float>(static_cast<double>(damp_rel) * mean_h);
    }
  }
}

__device__ __forceinline__ void decode_tri(int t, int& I, int& J) {
  int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= t) ++i;
  while (i * (i + 1) / 2 > t) --i;
  I = i;
  J = t - i * (i + 1) / 2;
}

// One 32 x 32 lower tile pair per CTA (blockDim 32 x 8).
__global__ void __launch_bounds__(256)
finalize_kernel(float* S_H, float* R, int64_t n, float scale, const float* lam_ptr) {
  __shared__ float t[32][33];
  int I, J;
  decode_tri(blockIdx.x, I, J);
  const int i0 = I * 32, j0 = J * 32;
  const float lam = *lam_ptr;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    t[r][tx] = (i < n && j < n) ? S_H[i * n + j] * scale : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    if (I > J) {
      if (i < n && j < n) { S_H[i * n + j] = t[r][tx]; R[i * n + j] = t[r][tx]; }
      const int it = j0 + r, jt = i0 + tx;  // transposed position (upper tile)
      if (it < n && jt < n) { S_H[it * n + jt] = t[tx][r]; R[it * n + jt] = 0.f; }
    } else if (i < n && j < n) {
      const float h = (tx <= r) ? t[r][tx] : t[tx][r];
      S_H[i * n + j] = h;
      R[i * n + j] = (tx < r) ? h : (tx == r ? h + lam : 0.f);
    }
  }
}

// R = L2^T in place (L2 lower with zero upper): the result is upper with zero strict lower part.
__global__ void __launch_bounds__(256) transpose_to_upper_kernel(float* R, int64_t n) {
  __shared__ float t[32][33];
  int I, J;
  decode_tri(blockIdx.x, I, J);
  const int i0 = I * 32, j0 = J * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    t[r][tx] = (i < n && j < n) ? R[i * n + j] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    if (I > J) {
      const int it = j0 + r, jt = i0 + tx;
      if (it < n && jt < n) R[it * n + jt] = t[tx][r];
      const int i = i0 + r, j = j0 + tx;
      if (i < n && j < n) R[i * n + j] = 0.f;
    } else {
      const int i = i0 + r, j = j0 + tx;
      if (i < n && j < n) R[i * n + j] = (tx >= r) ? t[tx][r] : 0.f;
    }
  }
}

// Reversed route: H = (2/N) S mirrored into S_H as above, and the lower triangle of
// J H_d J (entry [a][b] = H_d[n-1-a][n-1-b]) into R with its strict upper part zeroed.
__global__ void __launch_bounds__(256)
finalize_reversed_kernel(float* S_H, float* R, int64_t n, float scale, const float* lam_ptr) {
  __shared__ float t[32][33];
  int I, J;
  decode_tri(blockIdx.x, I, J);
  const int i0 = I * 32, j0 = J * 32;
  const float lam = *lam_ptr;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t m = n - 1;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    t[r][tx] = (i < n && j < n) ? S_H[i * n + j] * scale : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    if (I > J) {
      const int i = i0 + r, j = j0 + tx;
      if (i < n && j < n) S_H[i * n + j] = t[r][tx];
      const int it = j0 + r, jt = i0 + tx;          // transposed position (upper tile of H)
      if (it < n && jt < n) {
        S_H[it * n + jt] = t[tx][r];
        R[(m - it) * n + (m - jt)] = t[tx][r];      // H[jt][it], now below the diagonal
      }
      if (i < n && j < n) R[(m - i) * n + (m - j)] = 0.f;
    } else {
      const int i = i0 + r, j = j0 + tx;
      if (i < n && j < n) {
        const float h = (tx <= r) ? t[r][tx] : t[tx][r];
        S_H[i * n + j] = h;
        R[(m - i) * n + (m - j)] = (tx > r) ? h : (tx == r ? h + lam : 0.f);
      }
    }
  }
}

// Reversed route, last step: R = J V J with V = (Vb + Vs) the lower triangular inverse (ld n);
// the result is upper, its strict lower part zeroed. One lower 32 x 32 tile of V per CTA.
__global__ void __launch_bounds__(256)
reverse_to_upper_kernel(float* R, const float* Vb, const float* Vs, int64_t n) {
  int I, J;
  decode_tri(blockIdx.x, I, J);
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t m = n - 1;
  for (int r = ty; r < 32; r += 8) {
    const int a = I * 32 + r, b = J * 32 + tx;
    if (a < n && b < n) {
      const float v = (a >= b) ? Vb[a * n + b] + Vs[a * n + b] : 0.f;
      R[(m - a) * n + (m - b)] = v;
    }
    if (I > J) {                                    // the mirrored tile lands below the diagonal
      const int a2 = J * 32 + r, b2 = I * 32 + tx;
      if (a2 < n && b2 < n) R[(m - a2) * n + (m - b2)] = 0.f;
    }
  }
}

// ------------------------------------------------------------------------------------------------
// S3/S5 diagonal block: Cholesky of A[k0:k0+nb, k0:k0+nb] on chip (lower; the block's strict upper
// part is zeroed in A) and the tf32 split of its triangular inverse into (Db, Ds) with ld ldd.
// Blocked by 32: warp 0 factors each 32 x 32 diagonal piece with its rows in registers (the pivot
// column is shared through shared memory, pivots use rsqrt and their reciprocals are kept), then
// inverts the piece while warps 1-3 solve the rows below it by forward substitution; all warps
// update the trailing part. The off-diagonal pieces of the inverse follow from
// X[bi][bj] = -X[bi][bi] * sum_k L[bi][k] X[k][bj]. A pivot that is not positive records
// info_base + k0 + j + 1 (or, for a factorization of the order-reversed matrix of order rev_n > 0,
// the 1-based index of that pivot in the original order, rev_n - k0 - j) and is replaced by 1 so
// the remaining arithmetic stays finite.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(la::kDiagThreads)
potrf_diag_kernel(float* A, int64_t lda, int k0, int nb, float* Db, float* Ds, int64_t ldd,
                  int32_t* info, int info_base, int rev_n) {
  constexpr int NB = 128, LD = 129;
  extern __shared__ float sm[];
  float* L = sm;
  float* X = sm + NB * LD;
  float* T = sm + 2 * NB * LD;     // [3][32][33]
  __shared__ float rdiag[NB];      // 1 / L[j][j]
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = 16;
  if (tid == 0) bad = -1;
  const bool vec = ((lda & 3) == 0) && ((k0 & 3) == 0) && ((ldd & 3) == 0) &&
                   ((reinterpret_cast<uintptr_t>(A) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Db) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Ds) & 15) == 0);
#pragma unroll 4
  for (int e = tid; e < NB * NB / 4; e += 512) {
    const int i = e >> 5, j = (e & 31) * 4;
    float v[4];
    if (vec && i < nb && j + 3 < nb) {
      const float4 q = *reinterpret_cast<const float4*>(A + (k0 + i) * lda + k0 + j);
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = (i < nb && j + u < nb) ? A[(k0 + i) * lda + k0 + j + u] : (i == j + u ? 1.f : 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) L[i * LD + j + u] = (j + u <= i) ? v[u] : 0.f;
  }
  __syncthreads();
  for (int kb = 0; kb < 4; ++kb) {
    const int c0 = kb * 32;
    if (warp == 0) {
      // lane l owns row c0 + l of the 32 x 32 piece, in registers; the pivot column goes through
      // shared memory (double-buffered, one warp sync per pivot) so each step reads it with
      // broadcast loads; pivot reciprocals stay in registers until the piece is done
      float d[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) d[k] = L[(c0 + lane) * LD + c0 + k];
      float* col = T;  // 2 x 32-float scratch
      float rr = 0.f;
      int badj = 32;
#pragma unroll 32
      for (int j = 0; j < 32; ++j) {
        const float piv = __shfl_sync(0xffffffffu, d[j], j);
        const bool ok = piv > 0.f && piv < INFINITY;
        const float r = ok ? rsqrtf(piv) : 1.f;
        badj = (!ok && badj == 32) ? j : badj;
        rr = (lane == j) ? r : rr;
        const float a = (lane == j) ? (ok ? piv * r : 1.f) : (lane > j ? d[j] * r : 0.f);
        d[j] = a;
        col[(j & 1) * 32 + lane] = a;
        __syncwarp();
#pragma unroll 32
        for (int k = 0; k < 32; ++k)
          if (k > j && lane >= k) d[k] = fmaf(-a, col[(j & 1) * 32 + k], d[k]);
      }
      rdiag[c0 + lane] = rr;
      if (lane == 0 && badj < 32 && bad < 0) bad = c0 + badj;
#pragma unroll
      for (int k = 0; k < 32; ++k) L[(c0 + lane) * LD + c0 + k] = (k <= lane) ? d[k] : 0.f;
    }
    __syncthreads();
    if (warp == 0) {
      // inverse of the piece: lane t computes column t
      float x[32];
#pragma unroll 32
      for (int i = 0; i < 32; ++i) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll 32
        for (int m = 0; m < 32; m += 2) {
          if (m < i && m >= lane) s0 = fmaf(L[(c0 + i) * LD + c0 + m], x[m], s0);
          if (m + 1 < i && m + 1 >= lane) s1 = fmaf(L[(c0 + i) * LD + c0 + m + 1], x[m + 1], s1);
        }
        x[i] = (i < lane) ? 0.f : (((i == lane) ? 1.f : 0.f) - (s0 + s1)) * rdiag[c0 + i];
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) X[(c0 + i) * LD + c0 + lane] = x[i];
    } else if (c0 + 32 + (warp - 1) * 32 < NB) {
      // panel below the piece: x P^T = a by forward substitution, lane = row
      const int r = c0 + 32 + (warp - 1) * 32 + lane;
      float x[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = L[r * LD + c0 + c];
#pragma unroll 32
      for (int c = 0; c < 32; ++c) {
        float s0 = x[c], s1 = 0.f;
#pragma unroll 32
        for (int m = 0; m < 32; m += 2) {
          if (m < c) s0 = fmaf(-x[m], L[(c0 + c) * LD + c0 + m], s0);
          if (m + 1 < c) s1 = fmaf(-x[m + 1], L[(c0 + c) * LD + c0 + m + 1], s1);
        }
        x[c] = (s0 + s1) * rdiag[c0 + c];
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) L[r * LD + c0 + c] = x[c];
    }
    __syncthreads();
    // trailing update: lane owns column l (panel values in registers); rows i >= l in steps of 4,
    // two rows at a time
    {
      const int base = c0 + 32;
      const int ncol = NB - base;
      for (int t = warp * 32; t < ncol * 4; t += NW * 32) {
        const int item = t + lane;
        if (item < ncol * 4) {
          const int l = base + item % ncol;
          const int g = item / ncol;
          float pv[32];
#pragma unroll
          for (int m = 0; m < 32; ++m) pv[m] = L[l * LD + c0 + m];
          int i = l + g;
          for (; i + 4 < NB; i += 8) {
            float s0 = 0.f, s1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
            for (int m = 0; m < 32; m += 2) {
              s0 = fmaf(L[i * LD + c0 + m], pv[m], s0);
              s1 = fmaf(L[i * LD + c0 + m + 1], pv[m + 1], s1);
              u0 = fmaf(L[(i + 4) * LD + c0 + m], pv[m], u0);
              u1 = fmaf(L[(i + 4) * LD + c0 + m + 1], pv[m + 1], u1);
            }
            L[i * LD + l] -= s0 + s1;
            L[(i + 4) * LD + l] -= u0 + u1;
          }
          if (i < NB) {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int m = 0; m < 32; m += 2) {
              s0 = fmaf(L[i * LD + c0 + m], pv[m], s0);
              s1 = fmaf(L[i * LD + c0 + m + 1], pv[m + 1], s1);
            }
            L[i * LD + l] -= s0 + s1;
          }
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0 && bad >= 0 && bad < nb)
    record_info(info, rev_n > 0 ? rev_n - (k0 + bad) : info_base + k0 + bad + 1);
  // off-diagonal pieces of the inverse, 2 x 2 outputs per thread (rows r, r+16; cols c, c+16)
  for (int bi = 1; bi < 4; ++bi) {
    for (int e = tid; e < bi * 256; e += 512) {
      const int bj = e >> 8, r = (e >> 4) & 15, c = e & 15;
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
      const float* l0 = L + (32 * bi + r) * LD;
      const float* l1 = L + (32 * bi + r + 16) * LD;
      for (int k = 32 * bj; k < 32 * bi; ++k) {
        const float x0 = X[k * LD + 32 * bj + c], x1 = X[k * LD + 32 * bj + c + 16];
        const float p0 = l0[k], p1 = l1[k];
        a00 = fmaf(p0, x0, a00); a01 = fmaf(p0, x1, a01);
        a10 = fmaf(p1, x0, a10); a11 = fmaf(p1, x1, a11);
      }
      float* t = T + bj * 32 * 33;
      t[r * 33 + c] = a00; t[r * 33 + c + 16] = a01;
      t[(r + 16) * 33 + c] = a10; t[(r + 16) * 33 + c + 16] = a11;
    }
    __syncthreads();
    for (int e = tid; e < bi * 256; e += 512) {
      const int bj = e >> 8, r = (e >> 4) & 15, c = e & 15;
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
      const float* x0r = X + (32 * bi + r) * LD + 32 * bi;
      const float* x1r = X + (32 * bi + r + 16) * LD + 32 * bi;
      const float* t = T + bj * 32 * 33;
#pragma unroll 8
      for (int m = 0; m < 32; ++m) {
        const float t0 = t[m * 33 + c], t1 = t[m * 33 + c + 16];
        const float p0 = x0r[m], p1 = x1r[m];
        a00 = fmaf(p0, t0, a00); a01 = fmaf(p0, t1, a01);
        a10 = fmaf(p1, t0, a10); a11 = fmaf(p1, t1, a11);
      }
      float* xo = X + (32 * bi) * LD + 32 * bj;
      xo[r * LD + c] = -a00; xo[r * LD + c + 16] = -a01;
      xo[(r + 16) * LD + c] = -a10; xo[(r + 16) * LD + c + 16] = -a11;
    }
    __syncthreads();
  }
#pragma unroll 4
  for (int e = tid; e < NB * NB / 4; e += 512) {
    const int i = e >> 5, j = (e & 31) * 4;
    if (i >= nb) continue;
    float lv[4], bv[4], sv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int jj = j + u;
      lv[u] = (jj <= i) ? L[i * LD + jj] : 0.f;
      const float x = ((jj >> 5) <= (i >> 5)) ? X[i * LD + jj] : 0.f;
      bv[u] = tf32_rna(x);
      sv[u] = x - bv[u];
    }
    if (vec && j + 3 < nb) {
      *reinterpret_cast<float4*>(A + (k0 + i) * lda + k0 + j) = make_float4(lv[0], lv[1], lv[2], lv[3]);
      *reinterpret_cast<float4*>(Db + i * ldd + j) = make_float4(bv[0], bv[1], bv[2], bv[3]);
      *reinterpret_cast<float4*>(Ds + i * ldd + j) = make_float4(sv[0], sv[1], sv[2], sv[3]);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (j + u >= nb) continue;
        A[(k0 + i) * lda + k0 + j + u] = lv[u];
        Db[i * ldd + j + u] = bv[u];
        Ds[i * ldd + j + u] = sv[u];
      }
    }
  }
}

static gptq_status launch_potrf_diag(float* A, int64_t n, int k0, int nb, float* Db, float* Ds,
                                     int64_t ldd, int32_t* info, int info_base, int rev_n,
                                     cudaStream_t stream) {
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(potrf_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             la::kDiagSmem) != cudaSuccess)
      return GPTQ_ECUDA;
    attr_done = true;
  }
  potrf_diag_kernel<<<1, la::kDiagThreads, la::kDiagSmem, stream>>>(A, n, k0, nb, Db, Ds, ldd, info,
                                                                     info_base, rev_n);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

struct Split {
  float* b;
  float* s;
};

// Blocked right-looking Cholesky of A (n x n, lower, in place).
//   Lsp:  tf32 split of L's panels (n x n, ld n), written as the panels are solved;
//   Dsp:  where each diagonal block's inverse goes (ld ld_dinv): at block k0 of an n x n matrix
//         when per_block is set (the block diagonal of L^-1), else one shared 128 x 128 scratch;
//   Psp:  split of the current panel before its solve (n x 128);
//   rev_n: > 0 when A is the order-reversed matrix (pivot codes then name original columns).
static gptq_status potrf_blocked(float* A, int64_t n, Split Lsp, Split Dsp, int64_t ld_dinv,
                                 bool per_block, Split Psp, int32_t* info, int info_base,
                                 int rev_n, cudaStream_t stream) {
  using namespace la;
  for (int64_t k0 = 0; k0 < n; k0 += kNB) {
    const int nb = static_cast<int>(n - k0 < kNB ? n - k0 : kNB);
    const int64_t doff = per_block ? k0 * ld_dinv + k0 : 0;
    GPTQ_TRY(launch_potrf_diag(A, n, static_cast<int>(k0), nb, Dsp.b + doff, Dsp.s + doff, ld_dinv,
                               info, info_base, rev_n, stream));
    const int64_t m = n - k0 - nb;
    if (m == 0) break;
    float* A21 = A + (k0 + nb) * n + k0;
    GPTQ_TRY(launch_split_tf32(A21, n, m, nb, Psp.b, Psp.s, kNB, stream));
    // panel solve: L21 = A21 * Dinv^T, written to A and, split, to Lsp
    const int64_t loff = (k0 + nb) * n + k0;
    TcGemmArgs t{Psp.b, Psp.s, Dsp.b + doff, Dsp.s + doff, kNB, ld_dinv, 0, 0,
                 static_cast<int>(m), nb, nb, 1.f, 0.f, 0, 0, 0,
                 A21, n, Lsp.b + loff, Lsp.s + loff, n, info};
    GPTQ_TRY(launch_gemm_tc(t, stream));
    // trailing update: A22 -= L21 L21^T (lower tiles)
    TcGemmArgs u{Lsp.b + loff, Lsp.s + loff, Lsp.b + loff, Lsp.s + loff, n, n, 0, 0,
                 static_cast<int>(m), static_cast<int>(m), nb, -1.f, 1.f, 1, 0, 0,
                 A + (k0 + nb) * n + (k0 + nb), n, nullptr, nullptr, 0, info};
    GPTQ_TRY(launch_gemm_tc(u, stream));
  }
  return GPTQ_OK;
}

namespace {
struct PrepareWs {
  Split L, V, P, D;
  float* lam;
};

PrepareWs carve(void* ws, int64_t n) {
  using namespace la;
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](size_t bytes) {
    float* r = reinterpret_cast<float*>(p);
    p += align_up(bytes, 256);
    return r;
  };
  PrepareWs w;
  const size_t nn = static_cast<size_t>(n) * n * 4, np = static_cast<size_t>(n) * kNB * 4;
  w.L.b = take(nn); w.L.s = take(nn);
  w.V.b = take(nn); w.V.s = take(nn);
  w.P.b = take(np); w.P.s = take(np);
  w.D.b = take(kNB * kNB * 4); w.D.s = take(kNB * kNB * 4);
  w.lam = take(256);
  return w;
}
}  // namespace

// S4a: L^-1 (into the split V, whose 128 x 128 diagonal blocks already hold the inverses of L's
// diagonal blocks) by recursive doubling. For a diagonal block of size s1 + s2 split into halves,
//   [L11 0; L21 L22]^-1 = [V11 0; V21 V22],  V21 = -V22 (L21 V11),
// so once every block of size s is inverted, all blocks of size 2s follow from two batched
// products (all merges of one level at once; a last, shorter merge separately):
//   T^T = V11^T L21^T   (s x s2; V11 lower, so k starts at the tile's row),
//   V21 = -V22 T         (s2 x s; V22 lower, so k stops after the tile's rows).
// T^T is kept in V's strict upper triangle at [o : o+s, o+s : o+s+s2], which nothing else reads.
static gptq_status trtri_merge(const PrepareWs& w, int64_t n, int64_t o, int64_t s1, int64_t s2,
                               int batch, int32_t* info, cudaStream_t stream) {
  const int64_t t_off = o * n + o + s1;               // T^T block
  const int64_t v21_off = (o + s1) * n + o;           // V21 block
  TcGemmArgs t{w.V.b + o * n + o, w.V.s + o * n + o, w.L.b + (o + s1) * n + o,
               w.L.s + (o + s1) * n + o, n, n, 1, 0,
               static_cast<int>(s1), static_cast<int>(s2), static_cast<int>(s1), 1.f, 0.f, 0, 1, 0,
               nullptr, 0, w.V.b + t_off, w.V.s + t_off, n, info};
  t.batch = batch;
  t.bstride = 2 * s1;
  GPTQ_TRY(launch_gemm_tc(t, stream));
  TcGemmArgs u{w.V.b + (o + s1) * n + o + s1, w.V.s + (o + s1) * n + o + s1, w.V.b + t_off,
               w.V.s + t_off, n, n, 0, 0,
               static_cast<int>(s2), static_cast<int>(s1), static_cast<int>(s2), -1.f, 0.f, 0, 0, 0,
               nullptr, 0, w.V.b + v21_off, w.V.s + v21_off, n, info};
  u.batch = batch;
  u.bstride = 2 * s1;
  u.khi_from_m = 1;
  return launch_gemm_tc(u, stream);
}

static gptq_status trtri_doubling(const PrepareWs& w, int64_t n, int32_t* info,
                                  cudaStream_t stream) {
  for (int64_t s = la::kNB; s < n; s *= 2) {
    const int64_t full = n / (2 * s);                 // merges whose halves are both s wide
    if (full > 0) GPTQ_TRY(trtri_merge(w, n, 0, s, s, static_cast<int>(full), info, stream));
    const int64_t o = full * 2 * s;
    if (o + s < n) GPTQ_TRY(trtri_merge(w, n, o, s, n - o - s, 1, info, stream));
  }
  return GPTQ_OK;
}

size_t prepare_workspace_bytes(int64_t cols) {
  const size_t n = static_cast<size_t>(cols);
  return 4 * align_up(n * n * 4, 256) + 2 * align_up(n * la::kNB * 4, 256) +
         2 * align_up(la::kNB * la::kNB * 4, 256) + 256;
}

gptq_status run_prepare_hinv(float* S_H, float* R, int64_t n, int64_t n_total, float damp_rel,
                             int route, void* ws, int32_t* info, cudaStream_t stream) {
  using namespace la;
  PrepareWs w = carve(ws, n);

  // S2
  const double scale = 2.0 / static_cast<double>(n_total);
  diag_lambda_kernel<<<1, 1024, 0, stream>>>(S_H, n, scale, damp_rel, w.lam, info);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return GPTQ_ECUDA;
  const int nt = static_cast<int>((n + 31) / 32);
  const int ntri = nt * (nt + 1) / 2;
  const bool reversed = route != GPTQ_ROUTE_THREE_STEP;
  if (reversed)
    finalize_reversed_kernel<<<ntri, dim3(32, 8), 0, stream>>>(S_H, R, n, static_cast<float>(scale),
                                                               w.lam);
  else
    finalize_kernel<<<ntri, dim3(32, 8), 0, stream>>>(S_H, R, n, static_cast<float>(scale), w.lam);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return GPTQ_ECUDA;

  // S3: H_d = L L^T in R (reversed route: J H_d J = M M^T, M written as L below); the inverses of
  // L's diagonal blocks land in V (the split of L^-1)
  GPTQ_TRY(potrf_blocked(R, n, w.L, w.V, n, true, w.P, info, 0, reversed ? static_cast<int>(n) : 0,
                         stream));

  // S4a: the rest of L^-1 by recursive doubling over the diagonal blocks already inverted.
  GPTQ_TRY(trtri_doubling(w, n, info, stream));

  if (reversed) {
    // R = J M^-1 J
    reverse_to_upper_kernel<<<ntri, dim3(32, 8), 0, stream>>>(R, w.V.b, w.V.s, n);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
  }

  // S4b: H_d^-1 = L^-T L^-1 (lower tiles) into R
  TcGemmArgs h{w.V.b, w.V.s, w.V.b, w.V.s, n, n, 1, 1,
               static_cast<int>(n), static_cast<int>(n), static_cast<int>(n), 1.f, 0.f, 1, 1, 0,
               R, n, nullptr, nullptr, 0, info};
  GPTQ_TRY(launch_gemm_tc(h, stream));

  // S5: H_d^-1 = L2 L2^T (reusing the L split and the diagonal scratch), then R = L2^T
  GPTQ_TRY(potrf_blocked(R, n, w.L, w.D, kNB, false, w.P, info, static_cast<int>(n), 0, stream));
  transpose_to_upper_kernel<<<ntri, dim3(32, 8), 0, stream>>>(R, n);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

}  // namespace gptq
