// The 128 x 128 diagonal block of the blocked Cholesky (S3/S5), factored and inverted on chip by
// one CTA of 512 threads. Used by the standalone diagonal-block kernel and by the fused
// factorization step, whose first CTA factors the next diagonal block.
//
// "GPTQ second-order quantization" blog, "3. Cholesky reformulation"; "Part 3: Adaptive Rounding:
// GPTQ", "Algorithm GPTQ".
#pragma once

#include <climits>
#include <cmath>

#include "common.cuh"

namespace gptq {

namespace la {
constexpr int kNB = 128;       // panel / diagonal block width
constexpr int kLd = kNB + 1;   // padded shared-memory row
constexpr int kDiagThreads = 512;
constexpr int kDiagSmem = (2 * kNB * kLd + 3 * 32 * 100) * 4;
}  // namespace la

__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ void decode_tri(int t, int& I, int& J) {
  int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= t) ++i;
  while (i * (i + 1) / 2 > t) --i;
  I = i;
  J = t - i * (i + 1) / 2;
}

// ------------------------------------------------------------------------------------------------
// S3/S5 diagonal block: Cholesky of A[k0:k0+nb, k0:k0+nb] on chip (lower; the block's strict upper
// part is zeroed in A when store_l is set) and the tf32 split of its triangular inverse into
// (Db, Ds) with ld ldd. Blocked by 32-column pieces; for each piece kb:
//  F  warps 0-3 factor the piece and build its inverse in the same loop, eight columns per step
//     (factor_piece8_mw).
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

// Factor and invert one 32 x 32 piece, eight columns per step, on warps 0-3. Lane l is row l; each
// register holds L[l][k] for k < l (the factor's row) or the running sum for X[k][l] for k > l (the
// inverse's column, X[j][t] = (delta_jt - sum_{m<j} L[j][m] X[m][t]) / L[j][j]); the diagonal
// pair L[l][l], X[l][l] ends in ldiag / xdiag. Warp w keeps columns 8w .. 8w+7 of every row in
// e[0..7] and owns step w: it factors the step's 8 x 8 diagonal block itself (broadcast by
// shuffles), solves every row's eight entries of L or X and publishes them (A8, X8: two float4
// per row); after a barrier of the four warps each later warp applies them to its own columns:
// entries of L take -L[l][j] L[k][j] and entries of X take L[k][j] X[j][l], one FMA per register
// and column for both. A pivot that is not positive is replaced by 1 and its index goes to badj.
// (Four columns per step, eight steps, measured 7.4 k cycles for the first piece; this form 6.9 k.)
// ldiag / xdiag are valid in the warp that owns column `lane`.
__device__ __forceinline__ void factor_piece8_mw(float (&e)[8], float& ldiag, float& xdiag,
                                                 int& badj, float4* A8, float4* X8, int warp,
                                                 int lane) {
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int j = 8 * t;
    if (warp == t) {
      float b[8][8];
#pragma unroll
      for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int q = 0; q <= p; ++q) b[p][q] = __shfl_sync(0xffffffffu, e[q], j + p);
      float lb[8][8], r[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float d = b[q][q];
#pragma unroll
        for (int s = 0; s < q; ++s) d = fmaf(-lb[q][s], lb[q][s], d);
        const bool ok = d > 0.f && d < INFINITY;
        r[q] = ok ? rsqrtf(d) : 1.f;
        lb[q][q] = ok ? d * r[q] : 1.f;
        badj = (!ok && badj == 32) ? j + q : badj;
#pragma unroll
        for (int p = q + 1; p < 8; ++p) {
          float v = b[p][q];
#pragma unroll
          for (int s = 0; s < q; ++s) v = fmaf(-lb[p][s], lb[q][s], v);
          lb[p][q] = v * r[q];
        }
      }
      float a[8], x[8];                    // L[lane][j+q] and X[j+q][lane]
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = j + q;
        float sa = e[q], sx = -e[q];
#pragma unroll
        for (int s = 0; s < q; ++s) {
          sa = fmaf(-a[s], lb[q][s], sa);
          sx = fmaf(-lb[q][s], x[s], sx);
        }
        if (lane > k) {
          a[q] = sa * r[q];
          x[q] = 0.f;
          e[q] = a[q];
        } else if (lane == k) {
          a[q] = lb[q][q];
          x[q] = r[q];
          ldiag = lb[q][q];
          xdiag = r[q];
        } else {
          a[q] = 0.f;
          x[q] = sx * r[q];
          e[q] = x[q];
        }
      }
      A8[(t * 32 + lane) * 2] = make_float4(a[0], a[1], a[2], a[3]);
      A8[(t * 32 + lane) * 2 + 1] = make_float4(a[4], a[5], a[6], a[7]);
      X8[(t * 32 + lane) * 2] = make_float4(x[0], x[1], x[2], x[3]);
      X8[(t * 32 + lane) * 2 + 1] = make_float4(x[4], x[5], x[6], x[7]);
    }
    named_barrier_or(la::kFactorBar, 128, false);
    if (warp > t) {
      const float4 a0 = A8[(t * 32 + lane) * 2], a1 = A8[(t * 32 + lane) * 2 + 1];
      const float4 x0 = X8[(t * 32 + lane) * 2], x1 = X8[(t * 32 + lane) * 2 + 1];
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = 8 * warp + q;
        const float4 c0 = A8[(t * 32 + k) * 2], c1 = A8[(t * 32 + k) * 2 + 1];
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const bool fac = lane >= k;
#pragma unroll
        for (int u = 0; u < 8; ++u) e[q] = fmaf(cv[u], fac ? -av[u] : xv[u], e[q]);
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


// Load the block A[k0:k0+nb, k0:k0+nb] (ld lda) into L (ld kLd): lower part, strict upper part
// zero, identity outside nb. All 512 threads.
__device__ __forceinline__ void diag_load_block(float* L, const float* A, int64_t lda, int k0,
                                                int nb, bool vec) {
  constexpr int LD = la::kLd;
  const int tid = threadIdx.x;
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
}

// Store rows [i0, i1) of the block: L when asked, and the tf32 split of the inverse (only its row
// block and the ones left of it are nonzero). A warp per row (warps w0 .. w0 + nw - 1), the lanes
// along it, so the shared-memory reads are conflict-free and every store covers 128 bytes.
__device__ __forceinline__ void diag_store_rows(const float* L, const float* X, int i0, int i1,
                                                int w0, int nw, float* A, int64_t lda, int k0,
                                                int nb, float* Db, float* Ds, int64_t ldd,
                                                int store_l) {
  constexpr int NB = 128, LD = la::kLd;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = i0 + (warp - w0); i < i1 && i < nb; i += nw) {
#pragma unroll
    for (int u = 0; u < NB / 32; ++u) {
      const int c = 32 * u + lane;
      if (c < nb) {
        const float x = (u <= (i >> 5)) ? X[i * LD + c] : 0.f;
        const float bx = tf32_rna(x);
        if (store_l) A[(k0 + i) * lda + k0 + c] = (c <= i) ? L[i * LD + c] : 0.f;
        Db[i * ldd + c] = bx;
        Ds[i * ldd + c] = x - bx;
      }
    }
  }
}

// Factor and invert the block held in L (as diag_load_block leaves it): the tf32 split of its
// inverse goes to (Db, Ds) with ld ldd, L itself to A[k0.., k0..] when store_l. stepA / stepX
// (256 float4 each) and `bad` are shared scratch; the first pivot that was not positive is
// recorded in info (see above). All 512 threads; starts and ends with every thread past a block
// barrier.
__device__ __forceinline__ void diag_factor_block(float* sm, float4* stepA, float4* stepX,
                                                  int* bad_sh, float* A, int64_t lda, int k0,
                                                  int nb, float* Db, float* Ds, int64_t ldd,
                                                  int32_t* info, int info_base, int rev_n,
                                                  int store_l) {
  constexpr int NB = 128, LD = la::kLd, LDT = la::kLdt;
  float* L = sm;
  float* X = sm + NB * LD;
  float* PT = sm + 2 * NB * LD;    // [32][LDT]: the panel below the piece, transposed
  float* OT = PT + 32 * LDT;       // 2 x [32][LDT]: partial sums of inverse row blocks
  int& bad = *bad_sh;              // first pivot that was not positive (INT_MAX: none)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad = INT_MAX;
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
      factor_piece8_mw(e, ldiag, xdiag, badj, stepA, stepX, warp, lane);
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
      // row blocks 0-2 of the inverse (and rows 0-95 of L) are final now: store them while the
      // last piece is factored
      if (kb == 3) diag_store_rows(L, X, 0, 96, 4, 12, A, lda, k0, nb, Db, Ds, ldd, store_l);
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
  // the last row block (rows 96 ..; the others were stored alongside the last piece)
  diag_store_rows(L, X, 96, NB, 0, la::kDiagThreads / 32, A, lda, k0, nb, Db, Ds, ldd, store_l);
}

}  // namespace gptq
