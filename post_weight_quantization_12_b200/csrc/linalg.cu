// S2-S5 -- from the accumulated S to the upper factor R of the damped inverse Hessian.
//
// "GPTQ second-order quantization" blog, "The objective is layer output" (H = 2 X X^T) and
// "3. Cholesky reformulation" (damping about 1 % of the mean diagonal; one Cholesky up front);
// "Part 3: Adaptive Rounding: GPTQ", "Observation 3" and "Algorithm GPTQ" (Cholesky of H^-1,
// whose rows are read during quantization).
//
// Two routes to the same R (the upper factor with positive diagonal is unique):
//  * three-step, as the pages write it: H_d = L L^T (blocked right-looking Cholesky, 128-wide
//    panels), L^-1 (triangular inverse by recursive doubling), H_d^-1 = L^-T L^-1
//    (triangular product, lower half only), H_d^-1 = L2 L2^T (second Cholesky), R = L2^T;
//  * reversed: with J the order-reversing permutation, J H_d J = M M^T (one Cholesky), so
//    H_d = U U^T with U = J M J upper, H_d^-1 = U^-T U^-1 and R = U^-1 = J M^-1 J: one Cholesky
//    and one triangular inverse, half the flops and half the chain of diagonal blocks.
// Each 128 x 128 diagonal block is factored and inverted on chip by one CTA; everything else is a
// 3xTF32 tensor-core matrix product whose operands are kept as tf32 (big, small) pairs in the
// workspace.
#include <climits>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace la {
constexpr int kNB = 128;       // panel / diagonal block width
constexpr int kLd = kNB + 1;   // padded shared-memory row
constexpr int kDiagThreads = 512;
constexpr int kDiagSmem = (2 * kNB * kLd + 3 * 32 * 100) * 4;
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
  griddep_wait();
  griddep_launch_dependents();

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
  griddep_wait();
  griddep_launch_dependents();

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
  griddep_wait();
  griddep_launch_dependents();

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
  griddep_wait();
  griddep_launch_dependents();

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
  griddep_wait();
  griddep_launch_dependents();

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
// part is zeroed in A when store_l is set) and the tf32 split of its triangular inverse into
// (Db, Ds) with ld ldd. Blocked by 32-column pieces; for each piece kb:
//  F  warps 0-3 factor the piece and build its inverse in the same loop, four columns per step
//     (factor_piece4_mw).
//     Meanwhile warps 4-15 finish the previous piece's trailing update beyond this piece's
//     columns and form the block's inverse row blocks,
//     X[b][j] = -X[b][b] * sum_m L[b][m] X[m][j]: the sum for row block kb and the product with
//     X[kb-1][kb-1] for row block kb-1.
//  S  rows below the piece: L21 = A21 X_kk^T, 4 x 4 register tiles, written transposed into PT;
//  T  trailing update A22 -= L21 L21^T on lower 4 x 4 tiles read from PT as float4, while PT is
//     copied back into the panel columns of L.
// A pivot that is not positive records info_base + k0 + j + 1 (or, for a factorization of the
// order-reversed matrix of order rev_n > 0, the 1-based index of that pivot in the original
// order, rev_n - k0 - j) and is replaced by 1 so the remaining arithmetic stays finite.
// ------------------------------------------------------------------------------------------------
namespace la {
constexpr int kLdt = 100;      // PT / OT row: 96 entries + pad, a multiple of 4 for float4 access
constexpr int kInverseBar = 1, kFactorBar = 2;
constexpr int kInverseThreads = kDiagThreads - 128;
}

// First half of row block b of the inverse: OT[r][j] = sum_m L[32b + r][m] X[m][j], j < 32b, over
// the row blocks already inverted. Threads first .. first + 64b - 1 take part (4 x 4 tiles).
__device__ __forceinline__ void inverse_row_sum(const float* L, const float* X, float* OT, int b,
                                                int first) {
  constexpr int LD = la::kLd, LDT = la::kLdt;
  const int t = threadIdx.x - first;
  if (t < 0 || t >= 64 * b) return;
  const int rg = t & 7, jg = t >> 3;
  const int r0 = 32 * b + 4 * rg;
  float acc[4][4] = {};
  for (int m = 32 * (jg >> 3); m < 32 * b; ++m) {
    float lv[4], xv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) lv[u] = L[(r0 + u) * LD + m];
#pragma unroll
    for (int v = 0; v < 4; ++v) xv[v] = X[m * LD + 4 * jg + v];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(lv[u], xv[v], acc[u][v]);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
    *reinterpret_cast<float4*>(OT + (4 * rg + u) * LDT + 4 * jg) =
        make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
}

// Second half: X[32b + r][j] = -sum_{m <= r} X[32b + r][32b + m] OT[m][j].
__device__ __forceinline__ void inverse_row_product(float* X, const float* OT, int b, int first) {
  constexpr int LD = la::kLd, LDT = la::kLdt;
  const int t = threadIdx.x - first;
  if (t < 0 || t >= 64 * b) return;
  const int rg = t & 7, jg = t >> 3;
  const int r0 = 32 * b + 4 * rg;
  float acc[4][4] = {};
  for (int m = 0; m < 4 * rg + 4; ++m) {         // X[b][b] is lower triangular
    float xb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) xb[u] = X[(r0 + u) * LD + 32 * b + m];
    const float4 o = *reinterpret_cast<const float4*>(OT + m * LDT + 4 * jg);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc[u][0] = fmaf(xb[u], o.x, acc[u][0]);
      acc[u][1] = fmaf(xb[u], o.y, acc[u][1]);
      acc[u][2] = fmaf(xb[u], o.z, acc[u][2]);
      acc[u][3] = fmaf(xb[u], o.w, acc[u][3]);
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) X[(r0 + u) * LD + 4 * jg + v] = -acc[u][v];
}

// Factor and invert one 32 x 32 piece, four columns per step, on warps 0-3. Lane l is row l; each
// register holds L[l][k] for k < l (the factor's row) or the running sum for X[k][l] for k > l (the
// inverse's column, X[j][t] = (delta_jt - sum_{m<j} L[j][m] X[m][t]) / L[j][j]); the diagonal
// pair L[l][l], X[l][l] ends in ldiag / xdiag. Per step the owning warp factors the step's 4 x 4
// diagonal block itself (broadcast by shuffles) and solves every row's four entries of L or X;
// entries of L then take -L[l][j] L[k][j] and entries of X take L[k][j] X[j][l], so one FMA per
// register and column serves both. A pivot that is not positive is replaced by 1 and its index
// goes to badj. Warp w keeps columns 8w .. 8w+7 of every row in e[0..7]; step t (columns
// 4t .. 4t+3) belongs to warp t/2, which publishes every row's entries of L (A4) and of X (X4) for
// the step; after a barrier of the four warps each warp applies them to its later columns.
// ldiag / xdiag are valid in the warp that owns column `lane`.
__device__ __forceinline__ void factor_piece4_mw(float (&e)[8], float& ldiag, float& xdiag,
                                                 int& badj, float4* A4, float4* X4, int warp,
                                                 int lane) {
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int j = 4 * t, q0 = (t & 1) * 4;
    if (warp == (t >> 1)) {
      float b[4][4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q <= p; ++q) b[p][q] = __shfl_sync(0xffffffffu, e[q0 + q], j + p);
      float lb[4][4], r[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float d = b[q][q];
#pragma unroll
        for (int s = 0; s < q; ++s) d = fmaf(-lb[q][s], lb[q][s], d);
        const bool ok = d > 0.f && d < INFINITY;
        r[q] = ok ? rsqrtf(d) : 1.f;
        lb[q][q] = ok ? d * r[q] : 1.f;
        badj = (!ok && badj == 32) ? j + q : badj;
#pragma unroll
        for (int p = q + 1; p < 4; ++p) {
          float v = b[p][q];
#pragma unroll
          for (int s = 0; s < q; ++s) v = fmaf(-lb[p][s], lb[q][s], v);
          lb[p][q] = v * r[q];
        }
      }
      float a[4], x[4];                    // L[lane][j+q] and X[j+q][lane]
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = j + q;
        float sa = e[q0 + q], sx = -e[q0 + q];
#pragma unroll
        for (int s = 0; s < q; ++s) {
          sa = fmaf(-a[s], lb[q][s], sa);
          sx = fmaf(-lb[q][s], x[s], sx);
        }
        if (lane > k) {
          a[q] = sa * r[q];
          x[q] = 0.f;
          e[q0 + q] = a[q];
        } else if (lane == k) {
          a[q] = lb[q][q];
          x[q] = r[q];
          ldiag = lb[q][q];
          xdiag = r[q];
        } else {
          a[q] = 0.f;
          x[q] = sx * r[q];
          e[q0 + q] = x[q];
        }
      }
      A4[t * 32 + lane] = make_float4(a[0], a[1], a[2], a[3]);
      X4[t * 32 + lane] = make_float4(x[0], x[1], x[2], x[3]);
    }
    named_barrier_or(la::kFactorBar, 128, false);
    if (warp >= (t >> 1)) {
      const float4 a4 = A4[t * 32 + lane], x4 = X4[t * 32 + lane];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = 8 * warp + q;
        if (k > j + 3) {
          const float4 c = A4[t * 32 + k];
          const bool fac = lane >= k;
          e[q] = fmaf(c.x, fac ? -a4.x : x4.x, e[q]);
          e[q] = fmaf(c.y, fac ? -a4.y : x4.y, e[q]);
          e[q] = fmaf(c.z, fac ? -a4.z : x4.z, e[q]);
          e[q] = fmaf(c.w, fac ? -a4.w : x4.w, e[q]);
        }
      }
    }
  }
}

// One lower 4 x 4 tile of the trailing update A22 -= L21 L21^T inside the diagonal block: rows
// c0 + 32 + 4 bi .., columns c0 + 32 + 4 bl .. (bl <= bi), the panel L21 read transposed from PT.
__device__ __forceinline__ void trailing_tile(const float* PT, float* L, int c0, int bi, int bl) {
  constexpr int LD = la::kLd, LDT = la::kLdt;
  float acc[4][4] = {};
#pragma unroll 8
  for (int m = 0; m < 32; ++m) {
    const float4 a4 = *reinterpret_cast<const float4*>(PT + m * LDT + 4 * bi);
    const float4 b4 = *reinterpret_cast<const float4*>(PT + m * LDT + 4 * bl);
    const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
  }
  const int i0 = c0 + 32 + 4 * bi, l0 = c0 + 32 + 4 * bl;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v)
      if (l0 + v <= i0 + u) L[(i0 + u) * LD + l0 + v] -= acc[u][v];
}

__global__ void __launch_bounds__(la::kDiagThreads)
potrf_diag_kernel(float* A, int64_t lda, int k0, int nb, float* Db, float* Ds, int64_t ldd,
                  int32_t* info, int info_base, int rev_n, int store_l) {
  griddep_wait();
  griddep_launch_dependents();

  constexpr int NB = 128, LD = la::kLd, LDT = la::kLdt;
  extern __shared__ float sm[];
  float* L = sm;
  float* X = sm + NB * LD;
  float* PT = sm + 2 * NB * LD;    // [32][LDT]: the panel below the piece, transposed
  float* OT = PT + 32 * LDT;       // 2 x [32][LDT]: partial sums of inverse row blocks
  __shared__ float4 stepA[256];    // per factor step: every row's four entries of L
  __shared__ float4 stepX[256];    // per factor step: every row's four entries of X
  __shared__ int bad;              // first pivot that was not positive (INT_MAX: none)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad = INT_MAX;
  const bool vec = ((lda & 3) == 0) && ((k0 & 3) == 0) && ((ldd & 3) == 0) &&
                   ((reinterpret_cast<uintptr_t>(A) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Db) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Ds) & 15) == 0);
  // load the block (outside nb: identity)
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float v[4][4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = tid + (half * 4 + it) * 512;
      const int i = e >> 5, j = (e & 31) * 4;
      if (vec && i < nb && j + 3 < nb) {
        const float4 q = *reinterpret_cast<const float4*>(A + (k0 + i) * lda + k0 + j);
        v[it][0] = q.x; v[it][1] = q.y; v[it][2] = q.z; v[it][3] = q.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[it][u] = (i < nb && j + u < nb) ? A[(k0 + i) * lda + k0 + j + u]
                                            : (i == j + u ? 1.f : 0.f);
      }
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = tid + (half * 4 + it) * 512;
      const int i = e >> 5, j = (e & 31) * 4;
#pragma unroll
      for (int u = 0; u < 4; ++u) L[i * LD + j + u] = (j + u <= i) ? v[it][u] : 0.f;
    }
  }
  __syncthreads();
#pragma unroll 1
  for (int kb = 0; kb < 4; ++kb) {
    const int c0 = kb * 32;
    if (warp < 4) {
      // ---- F: factor and invert the piece (warps 0-3) ----
      float e[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = 8 * warp + q;
        e[q] = (k <= lane) ? L[(c0 + lane) * LD + c0 + k] : 0.f;
      }
      float ldiag = 1.f, xdiag = 1.f;
      int badj = 32;
      factor_piece4_mw(e, ldiag, xdiag, badj, stepA, stepX, warp, lane);
      if (lane == 0 && badj < 32) atomicMin(&bad, c0 + badj);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = 8 * warp + q;
        L[(c0 + lane) * LD + c0 + k] = (k < lane) ? e[q] : (k == lane ? ldiag : 0.f);
        X[(c0 + k) * LD + c0 + lane] = (k > lane) ? e[q] : (k == lane ? xdiag : 0.f);
      }
    } else {
      // ---- alongside F (warps 4-15): the previous piece's trailing update beyond the columns
      // of this piece, then the inverse row blocks ----
      const int first = 128;
      if (kb >= 1) {
        const int pc0 = c0 - 32, pnb4 = (NB - pc0 - 32) / 4;   // previous piece's trailing region
        const int nrest = (pnb4 - 8) * (pnb4 - 7) / 2;        // lower tiles with bl >= 8
        for (int t = tid - first; t < nrest; t += la::kInverseThreads) {
          int bi, bl;
          decode_tri(t, bi, bl);
          trailing_tile(PT, L, pc0, bi + 8, bl + 8);
        }
      }
      if (kb >= 2) {
        inverse_row_product(X, OT + ((kb - 1) & 1) * 32 * LDT, kb - 1, first);
        named_barrier_or(la::kInverseBar, la::kInverseThreads, false);
      }
      if (kb >= 1) inverse_row_sum(L, X, OT + (kb & 1) * 32 * LDT, kb, first);
    }
    __syncthreads();
    const int nbelow = NB - c0 - 32;
    if (nbelow == 0) break;
    // ---- S: L21 = A21 X_kk^T into PT (transposed) ----
    {
      const int nrq = nbelow / 4;
      if (tid < nrq * 8) {
        const int cg = (tid >> 3) & 7, rq = (tid & 7) + 8 * (tid >> 6);
        const int rr = c0 + 32 + 4 * rq;
        float acc[4][4] = {};
        for (int m = 0; m < 4 * cg + 4; ++m) {   // X_kk[c][m] = 0 for m > c
          float av[4], xv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) av[u] = L[(rr + u) * LD + c0 + m];
#pragma unroll
          for (int v = 0; v < 4; ++v) xv[v] = X[(c0 + 4 * cg + v) * LD + c0 + m];
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], xv[v], acc[u][v]);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<float4*>(PT + (4 * cg + v) * LDT + 4 * rq) =
              make_float4(acc[0][v], acc[1][v], acc[2][v], acc[3][v]);
      }
    }
    __syncthreads();
    // ---- T: A22 -= L21 L21^T on the next piece's 32 columns (lower 4 x 4 tiles with bl < 8),
    // and PT back into L's panel columns; the tiles further right are left to warps 4-15 while
    // the next piece is factored ----
    {
      const int nb4 = nbelow / 4;
      for (int it = tid; it < nb4 * 8; it += 512) {
        const int bl = it & 7, bi = it >> 3;
        if (bi >= bl) trailing_tile(PT, L, c0, bi, bl);
      }
      for (int e = tid; e < nbelow * 32; e += 512) {
        const int r = e >> 5, c = e & 31;
        L[(c0 + 32 + r) * LD + c0 + c] = PT[c * LDT + r];
      }
    }
    __syncthreads();
  }
  if (tid == 0 && bad < nb)
    record_info(info, rev_n > 0 ? rev_n - (k0 + bad) : info_base + k0 + bad + 1);
  // the last row block of the inverse (its sums were formed alongside the last piece)
  inverse_row_product(X, OT + 1 * 32 * LDT, 3, 0);
  __syncthreads();
  // store: L when asked, and the tf32 split of the inverse
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
      if (store_l)
        *reinterpret_cast<float4*>(A + (k0 + i) * lda + k0 + j) =
            make_float4(lv[0], lv[1], lv[2], lv[3]);
      *reinterpret_cast<float4*>(Db + i * ldd + j) = make_float4(bv[0], bv[1], bv[2], bv[3]);
      *reinterpret_cast<float4*>(Ds + i * ldd + j) = make_float4(sv[0], sv[1], sv[2], sv[3]);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (j + u >= nb) continue;
        if (store_l) A[(k0 + i) * lda + k0 + j + u] = lv[u];
        Db[i * ldd + j + u] = bv[u];
        Ds[i * ldd + j + u] = sv[u];
      }
    }
  }
}

static gptq_status launch_potrf_diag(float* A, int64_t n, int k0, int nb, float* Db, float* Ds,
                                     int64_t ldd, int32_t* info, int info_base, int rev_n,
                                     bool store_l, cudaStream_t stream) {
  const gptq_status st =
      set_max_dynamic_smem(reinterpret_cast<const void*>(potrf_diag_kernel), la::kDiagSmem);
  if (st != GPTQ_OK) return st;
  return launch_pdl(potrf_diag_kernel, dim3(1), dim3(la::kDiagThreads), la::kDiagSmem, stream, A, n,
                    k0, nb, Db, Ds, ldd, info, info_base, rev_n, store_l ? 1 : 0);
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
//   rev_n: > 0 when A is the order-reversed matrix (pivot codes then name original columns);
//   store_l: write the factored diagonal blocks back into A (only needed when A's own lower
//         triangle is the result; the panels below them are always written).
static gptq_status potrf_blocked(float* A, int64_t n, Split Lsp, Split Dsp, int64_t ld_dinv,
                                 bool per_block, Split Psp, int32_t* info, int info_base,
                                 int rev_n, bool store_l, cudaStream_t stream) {
  using namespace la;
  for (int64_t k0 = 0; k0 < n; k0 += kNB) {
    const int nb = static_cast<int>(n - k0 < kNB ? n - k0 : kNB);
    const int64_t doff = per_block ? k0 * ld_dinv + k0 : 0;
    GPTQ_TRY(launch_potrf_diag(A, n, static_cast<int>(k0), nb, Dsp.b + doff, Dsp.s + doff, ld_dinv,
                               info, info_base, rev_n, store_l, stream));
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
  GPTQ_TRY(launch_pdl(diag_lambda_kernel, dim3(1), dim3(1024), 0, stream, S_H, n, scale, damp_rel,
                      w.lam, info));
  const int nt = static_cast<int>((n + 31) / 32);
  const int ntri = nt * (nt + 1) / 2;
  const bool reversed = route != GPTQ_ROUTE_THREE_STEP;
  if (reversed)
    GPTQ_TRY(launch_pdl(finalize_reversed_kernel, dim3(ntri), dim3(32, 8), 0, stream, S_H, R, n,
                        static_cast<float>(scale), w.lam));
  else
    GPTQ_TRY(launch_pdl(finalize_kernel, dim3(ntri), dim3(32, 8), 0, stream, S_H, R, n,
                        static_cast<float>(scale), w.lam));

  // S3: H_d = L L^T in R (reversed route: J H_d J = M M^T, M written as L below); the inverses of
  // L's diagonal blocks land in V (the split of L^-1)
  GPTQ_TRY(potrf_blocked(R, n, w.L, w.V, n, true, w.P, info, 0, reversed ? static_cast<int>(n) : 0,
                         false, stream));

  // S4a: the rest of L^-1 by recursive doubling over the diagonal blocks already inverted.
  GPTQ_TRY(trtri_doubling(w, n, info, stream));

  if (reversed) {
    // R = J M^-1 J
    return launch_pdl(reverse_to_upper_kernel, dim3(ntri), dim3(32, 8), 0, stream, R, w.V.b, w.V.s,
                      n);
  }

  // S4b: H_d^-1 = L^-T L^-1 (lower tiles) into R
  TcGemmArgs h{w.V.b, w.V.s, w.V.b, w.V.s, n, n, 1, 1,
               static_cast<int>(n), static_cast<int>(n), static_cast<int>(n), 1.f, 0.f, 1, 1, 0,
               R, n, nullptr, nullptr, 0, info};
  GPTQ_TRY(launch_gemm_tc(h, stream));

  // S5: H_d^-1 = L2 L2^T (reusing the L split and the diagonal scratch), then R = L2^T
  GPTQ_TRY(potrf_blocked(R, n, w.L, w.D, kNB, false, w.P, info, static_cast<int>(n), 0, true,
                         stream));
  return launch_pdl(transpose_to_upper_kernel, dim3(ntri), dim3(32, 8), 0, stream, R, n);
}

}  // namespace gptq
