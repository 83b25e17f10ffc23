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
#include "diag_block.cuh"
#include "internal.h"

namespace gptq {

#define GPTQ_TRY(x)               \
  do {                            \
    gptq_status _s = (x);         \
    if (_s != GPTQ_OK) return _s; \
  } while (0)

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

__global__ void __launch_bounds__(la::kDiagThreads)
potrf_diag_kernel(float* A, int64_t lda, int k0, int nb, float* Db, float* Ds, int64_t ldd,
                  int32_t* info, int info_base, int rev_n, int store_l, int32_t* flags,
                  int n_flags) {
  griddep_wait();
  griddep_launch_dependents();

  extern __shared__ float sm[];
  __shared__ float4 stepA[256];    // per factor step: every row's four entries of L
  __shared__ float4 stepX[256];    // per factor step: every row's four entries of X
  __shared__ int bad;
  // the fused factorization's panel flags start from zero on every call
  for (int i = threadIdx.x; i < n_flags; i += blockDim.x) flags[i] = 0;
  const bool vec = ((lda & 3) == 0) && ((k0 & 3) == 0) &&
                   ((reinterpret_cast<uintptr_t>(A) & 15) == 0);
  diag_load_block(sm, A, lda, k0, nb, vec);
  diag_factor_block(sm, stepA, stepX, &bad, A, lda, k0, nb, Db, Ds, ldd, info, info_base, rev_n,
                    store_l);
}

static gptq_status launch_potrf_diag(float* A, int64_t n, int k0, int nb, float* Db, float* Ds,
                                     int64_t ldd, int32_t* info, int info_base, int rev_n,
                                     bool store_l, cudaStream_t stream, int32_t* flags = nullptr,
                                     int n_flags = 0) {
  const gptq_status st =
      set_max_dynamic_smem(reinterpret_cast<const void*>(potrf_diag_kernel), la::kDiagSmem);
  if (st != GPTQ_OK) return st;
  return launch_pdl(potrf_diag_kernel, dim3(1), dim3(la::kDiagThreads), la::kDiagSmem, stream, A, n,
                    k0, nb, Db, Ds, ldd, info, info_base, rev_n, store_l ? 1 : 0, flags, n_flags);
}

struct Split {
  float* b;
  float* s;
};

// Blocked right-looking Cholesky of A (n x n, lower, in place; n % 4 == 0, A 16-byte aligned),
// 128-wide blocks: the diagonal block 0 and the split of the first panel, then one fused launch
// per step (potrf_step.cu).
//   Lsp:   tf32 split of L's panels (n x n, ld n), written as the panels are solved;
//   Dsp:   where each diagonal block's inverse goes (ld ld_dinv): at block k0 of an n x n matrix
//          when per_block is set (the block diagonal of L^-1), else two 128 x 128 scratch blocks
//          used in turn;
//   Psp:   the split of the next panel, two n x 128 buffers used in turn (absolute rows);
//   flags: ceil(n / 128) ints, the steps' panel flags;
//   rev_n: > 0 when A is the order-reversed matrix (pivot codes then name original columns);
//   store_l: write L back into A (only needed when A's own lower triangle is the result).
static gptq_status potrf_blocked(float* A, int64_t n, Split Lsp, Split Dsp, int64_t ld_dinv,
                                 bool per_block, Split Psp, int32_t* flags, int32_t* info,
                                 int info_base, int rev_n, bool store_l, cudaStream_t stream) {
  using namespace la;
  const int T = static_cast<int>((n + kNB - 1) / kNB);
  const int nb0 = static_cast<int>(n < kNB ? n : kNB);
  GPTQ_TRY(launch_potrf_diag(A, n, 0, nb0, Dsp.b, Dsp.s, ld_dinv, info, info_base, rev_n, store_l,
                             stream, flags, T));
  if (T == 1) return GPTQ_OK;
  GPTQ_TRY(launch_split_tf32(A + kNB * n, n, n - kNB, kNB, Psp.b + kNB * kNB, Psp.s + kNB * kNB,
                             kNB, stream));
  return launch_potrf_fused(A, n, Lsp.b, Lsp.s, Dsp.b, Dsp.s, ld_dinv, per_block, Psp.b, Psp.s,
                            flags, info, info_base, rev_n, store_l, stream);
}

namespace {
struct PrepareWs {
  Split L, V, P, D;
  float* lam;
  int32_t* flags;
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
  const size_t nn = static_cast<size_t>(n) * n * 4, np = 2 * static_cast<size_t>(n) * kNB * 4;
  w.L.b = take(nn); w.L.s = take(nn);
  w.V.b = take(nn); w.V.s = take(nn);
  w.P.b = take(np); w.P.s = take(np);
  w.D.b = take(2 * kNB * kNB * 4); w.D.s = take(2 * kNB * kNB * 4);
  w.lam = take(256);
  w.flags = reinterpret_cast<int32_t*>(take(static_cast<size_t>((n + kNB - 1) / kNB) * 4));
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
  return 4 * align_up(n * n * 4, 256) + 2 * align_up(2 * n * la::kNB * 4, 256) +
         2 * align_up(2 * la::kNB * la::kNB * 4, 256) + 256 +
         align_up((n + la::kNB - 1) / la::kNB * 4, 256);
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
  GPTQ_TRY(potrf_blocked(R, n, w.L, w.V, n, true, w.P, w.flags, info, 0,
                         reversed ? static_cast<int>(n) : 0, false, stream));

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
  GPTQ_TRY(potrf_blocked(R, n, w.L, w.D, kNB, false, w.P, w.flags, info, static_cast<int>(n), 0,
                         true, stream));
  return launch_pdl(transpose_to_upper_kernel, dim3(ntri), dim3(32, 8), 0, stream, R, n);
}

}  // namespace gptq
