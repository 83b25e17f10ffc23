// S2-S5 -- from the accumulated S to the upper factor R of the damped inverse Hessian.
//
// "GPTQ second-order quantization" blog, "The objective is layer output" (H = 2 X X^T) and
// "3. Cholesky reformulation" (damping about 1 % of the mean diagonal; one Cholesky up front);
// "Part 3: Adaptive Rounding: GPTQ", "Observation 3" and "Algorithm GPTQ" (Cholesky of H^-1,
// whose rows are read during quantization).
//
// Route: H_d = L L^T (blocked right-looking Cholesky, 128-wide panels), L^-1 (blocked triangular
// inverse, row block by row block), H_d^-1 = L^-T L^-1 (triangular product, lower half only),
// H_d^-1 = L2 L2^T (second Cholesky), R = L2^T. Each 128 x 128 diagonal block is factored and
// inverted on chip by one CTA; everything else is a matrix product.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace la {
constexpr int kNB = 128;       // panel / diagonal block width
constexpr int kLd = kNB + 1;   // padded shared-memory row
constexpr int kDiagThreads = 512;
constexpr int kDiagSmem = 2 * kNB * kLd * 4;
}  // namespace la

// ------------------------------------------------------------------------------------------------
// fp32 matrix product (CUDA cores), 64 x 64 tiles, 4 x 4 outputs per thread.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gemm_f32_kernel(GemmArgs g) {
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (g.lower && n0 > m0 + 63) return;
  int klo = 0;
  if (g.klo_from_m) klo = max(klo, m0);
  if (g.klo_from_n) klo = max(klo, n0);
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (int k0 = klo; k0 < g.K; k0 += 16) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + r * 256;
      int mm, kk;
      if (g.transA) { kk = e >> 6; mm = e & 63; } else { mm = e >> 4; kk = e & 15; }
      const int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < g.M && k < g.K)
        v = g.transA ? g.A[static_cast<int64_t>(k) * g.lda + m] : g.A[static_cast<int64_t>(m) * g.lda + k];
      As[kk][mm] = v;
      int nn;
      if (g.transB) { nn = e >> 4; kk = e & 15; } else { kk = e >> 6; nn = e & 63; }
      const int n = n0 + nn, k2 = k0 + kk;
      float w = 0.f;
      if (n < g.N && k2 < g.K)
        w = g.transB ? g.B[static_cast<int64_t>(n) * g.ldb + k2] : g.B[static_cast<int64_t>(k2) * g.ldb + n];
      Bs[kk][nn] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = As[kk][ty * 4 + u]; b[u] = Bs[kk][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int m = m0 + ty * 4 + u;
    if (m >= g.M) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int n = n0 + tx * 4 + v;
      if (n >= g.N) continue;
      float* c = g.C + static_cast<int64_t>(m) * g.ldc + n;
      const float r = g.alpha * acc[u][v];
      *c = (g.beta != 0.f) ? fmaf(g.beta, *c, r) : r;
    }
  }
}

gptq_status launch_gemm_f32(const GemmArgs& g, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
  dim3 grid((g.N + 63) / 64, (g.M + 63) / 64);
  if (grid.y > 65535) return GPTQ_EUNSUPPORTED;
  gemm_f32_kernel<<<grid, 256, 0, stream>>>(g);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
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

// ------------------------------------------------------------------------------------------------
// S3/S5 diagonal block: Cholesky of A[k0:k0+nb, k0:k0+nb] in shared memory (lower; its strict upper
// part is zeroed in A) and the block's triangular inverse into Dinv (ld ldd). A pivot that is not
// positive records info_base + k0 + j + 1 and is replaced by 1 so the rest stays finite.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(la::kDiagThreads)
potrf_diag_kernel(float* A, int64_t lda, int k0, int nb, float* Dinv, int64_t ldd, int32_t* info,
                  int info_base) {
  using namespace la;
  extern __shared__ float sm[];
  float* L = sm;
  float* X = sm + kNB * kLd;
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  if (tid == 0) bad = -1;
  for (int e = tid; e < kNB * kNB; e += blockDim.x) {
    const int i = e / kNB, j = e % kNB;
    float v;
    if (i < nb && j < nb) v = (j <= i) ? A[(k0 + i) * lda + k0 + j] : 0.f;
    else v = (i == j) ? 1.f : 0.f;
    L[i * kLd + j] = v;
  }
  __syncthreads();
  for (int j = 0; j < kNB; ++j) {
    const float d = L[j * kLd + j];
    const bool ok = d > 0.f && d < INFINITY;
    const float ljj = ok ? sqrtf(d) : 1.f;
    if (!ok && tid == 0 && bad < 0) bad = j;
    const float inv = 1.f / ljj;
    for (int i = j + 1 + tid; i < kNB; i += blockDim.x) L[i * kLd + j] *= inv;
    __syncthreads();
    if (tid == 0) L[j * kLd + j] = ljj;
    for (int i = j + 1 + warp; i < kNB; i += nwarps) {
      const float lij = L[i * kLd + j];
      for (int l = j + 1 + lane; l <= i; l += 32) L[i * kLd + l] -= lij * L[l * kLd + j];
    }
    __syncthreads();
  }
  if (tid == 0 && bad >= 0 && bad < nb) record_info(info, info_base + k0 + bad + 1);
  // inverse by forward substitution on all columns at once: 4 threads per column
  {
    const int t = tid >> 2, part = tid & 3;
    for (int i = 0; i < kNB; ++i) {
      float s = 0.f;
      if (t < i)
        for (int m = t + part; m < i; m += 4) s = fmaf(L[i * kLd + m], X[m * kLd + t], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (part == 0) {
        float x = 0.f;
        if (t <= i) x = ((t == i ? 1.f : 0.f) - s) / L[i * kLd + i];
        X[i * kLd + t] = x;
      }
      __syncthreads();
    }
  }
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, j = e % nb;
    A[(k0 + i) * lda + k0 + j] = (j <= i) ? L[i * kLd + j] : 0.f;
    Dinv[i * ldd + j] = X[i * kLd + j];
  }
}

static gptq_status launch_potrf_diag(float* A, int64_t n, int k0, int nb, float* Dinv, int64_t ldd,
                                     int32_t* info, int info_base, cudaStream_t stream) {
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(potrf_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             la::kDiagSmem) != cudaSuccess)
      return GPTQ_ECUDA;
    attr_done = true;
  }
  potrf_diag_kernel<<<1, la::kDiagThreads, la::kDiagSmem, stream>>>(A, n, k0, nb, Dinv, ldd, info,
                                                                     info_base);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

#define GPTQ_TRY(x)                       \
  do {                                    \
    gptq_status _s = (x);                 \
    if (_s != GPTQ_OK) return _s;         \
  } while (0)

// Blocked right-looking Cholesky of A (n x n, lower, in place). The inverse of each diagonal block
// of L goes to dinv_dst + k0 * (ld_dinv + 1) when per_block_dst is set (so the block diagonal of
// L^-1 is produced for free), else to the same scratch block every panel.
static gptq_status potrf_blocked(float* A, int64_t n, float* dinv_base, int64_t ld_dinv,
                                 bool per_block_dst, float* panel, int32_t* info, int info_base,
                                 cudaStream_t stream) {
  using namespace la;
  for (int64_t k0 = 0; k0 < n; k0 += kNB) {
    const int nb = static_cast<int>(n - k0 < kNB ? n - k0 : kNB);
    float* dinv = per_block_dst ? dinv_base + k0 * ld_dinv + k0 : dinv_base;
    GPTQ_TRY(launch_potrf_diag(A, n, static_cast<int>(k0), nb, dinv, ld_dinv, info, info_base,
                               stream));
    const int64_t m = n - k0 - nb;
    if (m == 0) break;
    // panel solve: P = A21 * L11^-T = A21 * Dinv^T
    GemmArgs t{A + (k0 + nb) * n + k0, n, 0, dinv, ld_dinv, 1, panel, kNB,
               static_cast<int>(m), nb, nb, 1.f, 0.f, 0, 0, 0};
    GPTQ_TRY(launch_gemm_f32(t, stream));
    if (cudaMemcpy2DAsync(A + (k0 + nb) * n + k0, n * sizeof(float), panel, kNB * sizeof(float),
                          nb * sizeof(float), m, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
      return GPTQ_ECUDA;
    // trailing update: A22 -= P P^T (lower tiles)
    GemmArgs u{panel, kNB, 0, panel, kNB, 1, A + (k0 + nb) * n + (k0 + nb), n,
               static_cast<int>(m), static_cast<int>(m), nb, -1.f, 1.f, 1, 0, 0};
    GPTQ_TRY(launch_gemm_f32(u, stream));
  }
  return GPTQ_OK;
}

size_t prepare_workspace_bytes(int64_t cols) {
  const size_t n = static_cast<size_t>(cols);
  size_t b = align_up(n * n * 4, 256);             // L^-1
  b += align_up(n * la::kNB * 4, 256);             // panel / row-block scratch
  b += align_up(la::kNB * la::kNB * 4, 256);       // diagonal-block inverse scratch
  b += 256;                                        // lambda
  return b;
}

gptq_status run_prepare_hinv(float* S_H, float* R, int64_t n, int64_t n_total, float damp_rel,
                             void* ws, int32_t* info, cudaStream_t stream) {
  using namespace la;
  uint8_t* p = static_cast<uint8_t*>(ws);
  float* Linv = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(n) * n * 4, 256);
  float* panel = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(n) * kNB * 4, 256);
  float* dscratch = reinterpret_cast<float*>(p);
  p += align_up(kNB * kNB * 4, 256);
  float* lam = reinterpret_cast<float*>(p);

  // S2
  const double scale = 2.0 / static_cast<double>(n_total);
  diag_lambda_kernel<<<1, 1024, 0, stream>>>(S_H, n, scale, damp_rel, lam, info);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return GPTQ_ECUDA;
  const int nt = static_cast<int>((n + 31) / 32);
  const int ntri = nt * (nt + 1) / 2;
  finalize_kernel<<<ntri, dim3(32, 8), 0, stream>>>(S_H, R, n, static_cast<float>(scale), lam);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return GPTQ_ECUDA;

  // S3: H_d = L L^T in R; diagonal blocks of L^-1 straight into Linv
  GPTQ_TRY(potrf_blocked(R, n, Linv, n, true, panel, info, 0, stream));

  // S4a: rest of L^-1, row block by row block:
  //   Linv[i, :i] = -Linv[i, i] * (L[i, :i] * Linv[:i, :i])
  for (int64_t r0 = kNB; r0 < n; r0 += kNB) {
    const int rb = static_cast<int>(n - r0 < kNB ? n - r0 : kNB);
    GemmArgs t{R + r0 * n, n, 0, Linv, n, 0, panel, n, rb, static_cast<int>(r0),
               static_cast<int>(r0), 1.f, 0.f, 0, 0, 1};
    GPTQ_TRY(launch_gemm_f32(t, stream));
    GemmArgs u{Linv + r0 * n + r0, n, 0, panel, n, 0, Linv + r0 * n, n, rb, static_cast<int>(r0),
               rb, -1.f, 0.f, 0, 0, 0};
    GPTQ_TRY(launch_gemm_f32(u, stream));
  }

  // S4b: H_d^-1 = L^-T L^-1 (lower tiles) into R
  GemmArgs h{Linv, n, 1, Linv, n, 0, R, n, static_cast<int>(n), static_cast<int>(n),
             static_cast<int>(n), 1.f, 0.f, 1, 1, 0};
  GPTQ_TRY(launch_gemm_f32(h, stream));

  // S5: H_d^-1 = L2 L2^T, then R = L2^T
  GPTQ_TRY(potrf_blocked(R, n, dscratch, kNB, false, panel, info, static_cast<int>(n), stream));
  transpose_to_upper_kernel<<<ntri, dim3(32, 8), 0, stream>>>(R, n);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

}  // namespace gptq
