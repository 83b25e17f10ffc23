// S6-S8 -- the GPTQ column loop with lazy batch updates.
//
// "Part 3: Adaptive Rounding: GPTQ": "Observation 1" (one left-to-right column order shared by
// all rows, so rows run in parallel against one factor), "Observation 2: Lazy Batch Updates"
// (a block of B columns is processed on chip and the later columns get one matrix product per
// block), "Algorithm GPTQ"; the Vietnamese edition of the GPTQ blog, "2. Lazy batch update"
// (W[:, B:] -= E R[B, B:]); the design table and the blog's "Group-wise quantization"
// (asymmetric uniform grid per row or per group).
//
// Column loop layout: eight consecutive lanes own one weight row and hold the current block's values
// of that row in registers, four consecutive columns per lane per stretch of 32 columns. The
// block's B x B corner of R sits in shared memory. Every lane of a row computes the same codes for
// a sub-block of four columns from values broadcast by their owner lane, so one exchange serves
// four columns.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace gptq {

#define GPTQ_TRY_Q(x)             \
  do {                            \
    gptq_status _s = (x);         \
    if (_s != GPTQ_OK) return _s; \
  } while (0)


// tf32 rounding, for the (big, small) operand split of the trailing product
__device__ __forceinline__ float tf32_rna_q(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// Grid of the asymmetric min/max quantizer (IEEE float32, each step rounded once).
__device__ __forceinline__ void grid_params(float lo, float hi, float maxq, float& s, float& z) {
  lo = fminf(lo, 0.f);
  hi = fmaxf(hi, 0.f);
  if (lo == hi) { lo = -1.f; hi = 1.f; }
  s = __fdiv_rn(__fsub_rn(hi, lo), maxq);
  z = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), maxq);
}

// rint(w / s) with the quotient rounded once in IEEE float32, as the quantizer defines it, without a
// division in the common case: y = w * (1/s) is within ~2^-23 relative of the true quotient, so
// when y is farther than 1e-5 |y| from a half-integer, rint(y) equals rint(fl(w / s)); otherwise
// (rare) the correctly rounded division decides.
__device__ __forceinline__ float rint_quot(float w, float s, float inv_s) {
  const float y = w * inv_s;
  const float r = rintf(y);
  // |y - r| < 0.5 - 1e-5 (|y| + 1): a margin at least as wide as 1e-5 max(1, |y|)
  if (fabsf(y - r) < fmaf(-1e-5f, fabsf(y), 0.5f - 1e-5f)) return r;
  return rintf(__fdiv_rn(w, s));
}

// Quantizes the four columns of a sub-block in order: w4 holds their current values, rin[u][u2]
// = R[j0 + u][j0 + u2] (u2 > u) and idv[u] = 1 / R[j0 + u][j0 + u]. Each column's error is applied
// to the sub-block's later columns before they are quantized. Outputs, per column: the rounded
// quotient clamped to the grid (rc = q - z), the zero point z it used, the dequantized value and
// the error; and, in group mode, the grid of each column that starts a group of one or two
// columns (gs, gz).
// FAST: rint(w * (1/s)) with no branch; returns true if some quotient lies too near a half-integer
// for that product to decide its rounding -- the caller then redoes the sub-block with FAST =
// false, where rint_quot decides such columns by the correctly rounded division.
template <bool FAST, int MODE>
__device__ __forceinline__ bool quantize_sub_block(float (&w4)[4], const float (&rin)[3][4],
                                                   const float (&idv)[4], float& s, float& z,
                                                   float& inv_s, float maxq, int group, int j0,
                                                   float (&rc4)[4], float (&zq)[4],
                                                   float (&wh4)[4], float (&e4)[4],
                                                   float (&gs)[4], float (&gz)[4]) {
  bool near = false;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (MODE == 1 && group < 4 && ((j0 + u) & (group - 1)) == 0) {
      // a group of one or two columns starts here: its current values are in w4
      float lo = 0.f, hi = 0.f;
#pragma unroll
      for (int u2 = 0; u2 < 4; ++u2)
        if (u2 >= u && u2 < u + group) {
          lo = fminf(lo, w4[u2]);
          hi = fmaxf(hi, w4[u2]);
        }
      grid_params(lo, hi, maxq, s, z);
      inv_s = 1.f / s;
      gs[u] = s;
      gz[u] = z;
    }
    const float w = w4[u];
    float r;
    if (FAST) {
      const float y = w * inv_s;
      r = rintf(y);
      near |= !(fabsf(y - r) < fmaf(-1e-5f, fabsf(y), 0.5f - 1e-5f));
    } else {
      r = rint_quot(w, s, inv_s);
    }
    // clamp(r + z, 0, maxq) - z, exactly (small integers)
    const float rc = fminf(fmaxf(r, -z), maxq - z);
    const float wh = __fmul_rn(s, rc);
    const float e = __fmul_rn(__fsub_rn(w, wh), idv[u]);
    rc4[u] = rc;
    zq[u] = z;
    wh4[u] = wh;
    e4[u] = e;
#pragma unroll
    for (int u2 = u + 1; u2 < 4; ++u2) w4[u2] = fmaf(-e, rin[u][u2], w4[u2]);
  }
  return near;
}

// (a, a) as one 64-bit operand of the packed f32x2 instructions
__device__ __forceinline__ uint64_t pair_of(float a) {
  uint64_t p;
  asm("mov.b64 %0, {%1, %1};" : "=l"(p) : "f"(a));
  return p;
}

// (x0, x1) <- (a0 * b0 + x0, a1 * b1 + x1), one packed f32x2 fused multiply-add (each lane rounds
// once, as fmaf does)
__device__ __forceinline__ void fma_x2(float& x0, float& x1, uint64_t a2, float b0, float b1) {
  asm("{\n\t.reg .b64 b, c;\n\tmov.b64 b, {%3, %4};\n\tmov.b64 c, {%0, %1};\n\t"
      "fma.rn.f32x2 c, %2, b, c;\n\tmov.b64 {%0, %1}, c;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "l"(a2), "f"(b0), "f"(b1));
}

template <typename T>
__device__ __forceinline__ float load_w(const T* p);
template <>
__device__ __forceinline__ float load_w<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_w<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// bf16 rows of 8-element chunks (16-byte loads, two float4 stores); cols % 8 == 0, ldw % 8 == 0
__global__ void convert_bf16_vec_kernel(const __nv_bfloat16* __restrict__ W, int64_t ldw,
                                        float* __restrict__ Wh, int64_t rows, int64_t cols) {
  griddep_wait();
  griddep_launch_dependents();

  const int64_t c8 = cols / 8, total = rows * c8;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / c8, c = 8 * (e - r * c8);
    const uint4 raw = *reinterpret_cast<const uint4*>(W + r * ldw + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
    const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
    float4* dst = reinterpret_cast<float4*>(Wh + r * cols + c);
    dst[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
    dst[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
  }
}

template <typename T>
__global__ void convert_kernel(const T* __restrict__ W, int64_t ldw, float* __restrict__ Wh,
                               int64_t rows, int64_t cols) {
  griddep_wait();
  griddep_launch_dependents();

  const int64_t total = rows * cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    Wh[e] = load_w<T>(W + r * ldw + c);
  }
}

// One warp per row: grid of columns [c0, c0 + len) of the current weights.
__global__ void params_kernel(const float* __restrict__ Wh, int64_t rows, int64_t cols, int64_t c0,
                              int64_t len, int bits, float* scales, uint8_t* zeros, int G, int gi) {
  griddep_wait();
  griddep_launch_dependents();

  const int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float lo = 0.f, hi = 0.f;
  const float* w = Wh + row * cols + c0;
  for (int64_t c = lane; c < len; c += 32) {
    const float v = w[c];
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    float s, z;
    grid_params(lo, hi, static_cast<float>((1 << bits) - 1), s, z);
    scales[row * G + gi] = s;
    zeros[row * G + gi] = static_cast<uint8_t>(z);
  }
}

// One block of B columns [b0, b0 + nb) for every row. MODE 0: the grid is given per row
// (scales[row*G + gi_fixed]); MODE 1: groups of `group` columns (a power of two no wider than the
// block) start inside the block, and their grids are computed here from the current weights.
//
// TPR consecutive lanes own one row; lane `sub` holds the columns S t + 4 sub + u (S = 4 TPR,
// t < B/S, u < 4), so the lanes of a row cover each S-column stretch with one float4 each and their
// accesses to a row of R, W, E and the codes are contiguous. Columns go in sub-blocks of four,
// S t + 4o .. +3, owned by lane o: the row's lanes take the sub-block's current values from their
// owner, each quantizes the four columns itself (so one exchange serves four columns and nothing
// waits for a second exchange), and then each applies the four errors to its own later columns.
// Each weight therefore receives the updates of the earlier columns one sub-block at a time, in
// column order, with four fused multiply-adds per sub-block in the order of its columns.
//
// R is not written while a layer is quantized, so the block's B x B corner of R is fetched by
// bulk copies before the wait on the previous kernel (whose tail it overlaps). Only the entries
// right of the diagonal are used: updates are masked to later columns instead of relying on zeros
// below the diagonal.
template <int B, int MODE, int TPR>
__global__ void __launch_bounds__(128)
column_loop_kernel(float* __restrict__ Wh, int64_t rows, int64_t cols, const float* __restrict__ R,
                   int b0, int nb, int bits, int group, int gi_fixed, float* __restrict__ scales,
                   uint8_t* __restrict__ zeros, int G, uint8_t* __restrict__ codes,
                   float* __restrict__ Eb, float* __restrict__ Es, float* __restrict__ err_sq,
                   float* __restrict__ Rb_out, float* __restrict__ Rs_out, int64_t nrest,
                   int32_t* info) {
  constexpr int THREADS = 128;
  constexpr int S = 4 * TPR;       // columns covered by one float4 from each lane of a row
  constexpr int NT = B / S;        // float4 groups per lane
  constexpr int CPL = 4 * NT;      // columns per lane
  extern __shared__ __align__(128) float qsm[];
  float* Rz = qsm;                 // [B][B]: rows b0.. of R, columns b0.. (only k > i is read)
  float* inv_d = qsm + B * B;      // [B]: 1 / R[j][j]
  __shared__ __align__(8) uint64_t rbar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&rbar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // rows are 16-byte aligned and nb is a multiple of 4 (cols % 4 == 0, b0 % 4 == 0)
    mbar_arrive_expect_tx(&rbar, static_cast<uint32_t>(nb) * nb * 4u);
    for (int i = 0; i < nb; ++i)
      bulk_load(Rz + i * B, R + (b0 + i) * cols + b0, static_cast<uint32_t>(nb) * 4u, &rbar);
  }
  griddep_wait();
  griddep_launch_dependents();

  // the tf32 split of R[b0 : b0 + nb, b1 : cols] for the trailing product that follows this block,
  // spread over the whole grid (rows 16-byte aligned: cols % 4 == 0, b1 % 4 == 0)
  if (nrest > 0) {
    const int64_t b1 = b0 + nb, n4 = nrest / 4, total = nb * n4;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * THREADS;
    for (int64_t e0 = blockIdx.x * static_cast<int64_t>(THREADS) + threadIdx.x; e0 < total;
         e0 += 4 * stride) {
      float4 x[4];                         // four loads in flight
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t e = e0 + u * stride;
        if (e < total) {
          const int64_t i = e / n4, c = b1 + 4 * (e - i * n4);
          x[u] = *reinterpret_cast<const float4*>(R + (b0 + i) * cols + c);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t e = e0 + u * stride;
        if (e < total) {
          const int64_t i = e / n4, c = b1 + 4 * (e - i * n4);
          const float4 bg = make_float4(tf32_rna_q(x[u].x), tf32_rna_q(x[u].y),
                                        tf32_rna_q(x[u].z), tf32_rna_q(x[u].w));
          *reinterpret_cast<float4*>(Rb_out + i * cols + c) = bg;
          *reinterpret_cast<float4*>(Rs_out + i * cols + c) =
              make_float4(x[u].x - bg.x, x[u].y - bg.y, x[u].z - bg.z, x[u].w - bg.w);
        }
      }
    }
  }

  const int lane = threadIdx.x & 31;
  const int sub = lane & (TPR - 1);           // position within the row's lane group
  const int base_lane = lane & ~(TPR - 1);
  const int64_t row = blockIdx.x * static_cast<int64_t>(THREADS / TPR) + threadIdx.x / TPR;
  const bool valid = row < rows;

  auto colof = [&](int k) { return S * (k >> 2) + 4 * sub + (k & 3); };  // block column of v[k]

  float v[CPL];
  float qf[CPL];                  // codes of this lane's columns, converted when stored
  float err[CPL];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int c = S * t + 4 * sub;
    float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid && c < nb) w4 = *reinterpret_cast<const float4*>(Wh + row * cols + b0 + c);
    v[4 * t + 0] = w4.x; v[4 * t + 1] = w4.y; v[4 * t + 2] = w4.z; v[4 * t + 3] = w4.w;
  }
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    qf[k] = 0.f;
    err[k] = 0.f;
  }
  const float maxq = static_cast<float>((1 << bits) - 1);
  float s = 1.f, z = 0.f;
  if (MODE == 0 && valid) {
    s = scales[row * G + gi_fixed];
    z = static_cast<float>(zeros[row * G + gi_fixed]);
  }
  float inv_s = 1.f / s;

  // the corner of R has landed: the reciprocals of its diagonal
  if (!mbar_wait_bounded(&rbar, 0, &abort_flag, info)) {
    mbar_drain_bounded(&rbar, 0);            // let the copies in flight land before leaving
    return;
  }
  for (int i = threadIdx.x; i < nb; i += THREADS) inv_d[i] = 1.f / Rz[i * B + i];
  __syncthreads();

  // The stretch index t is unrolled (register indices must be constants); the sub-blocks of a
  // stretch run as a loop, which keeps the kernel small enough for the instruction cache.
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll 1
    for (int o = 0; o < TPR; ++o) {
      const int j0 = S * t + 4 * o;
      if (j0 >= nb) break;                   // nb % 4 == 0: sub-blocks are whole
      const bool own = (sub == o);
      float w4[4], e4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w4[u] = __shfl_sync(0xffffffffu, v[4 * t + u], base_lane + o);
      const float4 id4 = *reinterpret_cast<const float4*>(inv_d + j0);
      const float idv[4] = {id4.x, id4.y, id4.z, id4.w};
      float rin[3][4];                         // R[j0 + u][j0 .. j0 + 3], for the sub-block itself
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const float4 r4 = *reinterpret_cast<const float4*>(Rz + (j0 + u) * B + j0);
        rin[u][0] = r4.x; rin[u][1] = r4.y; rin[u][2] = r4.z; rin[u][3] = r4.w;
      }
      if (MODE == 1 && group >= 4 && (j0 & (group - 1)) == 0) {
        // a group of four or more columns starts here (at the sub-block's first column)
        float lo = 0.f, hi = 0.f;
        if (group == 4) {
#pragma unroll
          for (int u2 = 0; u2 < 4; ++u2) {
            lo = fminf(lo, w4[u2]);
            hi = fmaxf(hi, w4[u2]);
          }
        } else {
          // the row's lanes hold it
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const int c = colof(k);
            if (c >= j0 && c < j0 + group && c < nb) { lo = fminf(lo, v[k]); hi = fmaxf(hi, v[k]); }
          }
#pragma unroll
          for (int off = TPR / 2; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
          }
        }
        grid_params(lo, hi, maxq, s, z);
        inv_s = 1.f / s;
        if (valid && sub == 0) {
          const int gi = (b0 + j0) / group;
          scales[row * G + gi] = s;
          zeros[row * G + gi] = static_cast<uint8_t>(z);
        }
      }
      // the four columns, first with the branch-free rounding; if any quotient of the warp lies
      // near a half-integer, again from the same inputs with the exact decision
      float rc4[4], zq[4], wh4[4], gs[4], gz[4];
      {
        float w_in[4] = {w4[0], w4[1], w4[2], w4[3]};
        const float s0 = s, z0 = z, is0 = inv_s;
        const bool near = quantize_sub_block<true, MODE>(w4, rin, idv, s, z, inv_s, maxq, group,
                                                         j0, rc4, zq, wh4, e4, gs, gz);
        if (__any_sync(0xffffffffu, near)) {
          s = s0; z = z0; inv_s = is0;
          quantize_sub_block<false, MODE>(w_in, rin, idv, s, z, inv_s, maxq, group, j0, rc4, zq,
                                          wh4, e4, gs, gz);
        }
      }
      if (MODE == 1 && group < 4 && valid && sub == 0) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (((j0 + u) & (group - 1)) == 0) {
            const int gi = (b0 + j0 + u) / group;
            scales[row * G + gi] = gs[u];
            zeros[row * G + gi] = static_cast<uint8_t>(gz[u]);
          }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[4 * t + u] = own ? wh4[u] : v[4 * t + u];
        qf[4 * t + u] = own ? rc4[u] + zq[u] : qf[4 * t + u];
        err[4 * t + u] = own ? e4[u] : err[4 * t + u];
      }
      // the sub-block's errors on this lane's later columns (rank 4, one column after another),
      // two columns per packed multiply-add
      uint64_t ne2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) ne2[u] = pair_of(-e4[u]);
#pragma unroll
      for (int t2 = t; t2 < NT; ++t2) {
        if (t2 == t && sub <= o) continue;   // earlier columns, or the sub-block itself
        float4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          r[u] = *reinterpret_cast<const float4*>(Rz + (j0 + u) * B + S * t2 + 4 * sub);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          fma_x2(v[4 * t2 + 0], v[4 * t2 + 1], ne2[u], r[u].x, r[u].y);
          fma_x2(v[4 * t2 + 2], v[4 * t2 + 3], ne2[u], r[u].z, r[u].w);
        }
      }
    }
  }

  float sq = 0.f;
#pragma unroll
  for (int k = 0; k < CPL; ++k) sq = fmaf(err[k], err[k], sq);
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if (!valid) return;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int c = S * t + 4 * sub;
    if (c >= nb) continue;                   // nb % 4 == 0: a float4 is whole or absent
    float b4[4], s4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      b4[u] = tf32_rna_q(err[4 * t + u]);
      s4[u] = err[4 * t + u] - b4[u];
    }
    *reinterpret_cast<float4*>(Wh + row * cols + b0 + c) =
        make_float4(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]);
    *reinterpret_cast<float4*>(Eb + row * B + c) = make_float4(b4[0], b4[1], b4[2], b4[3]);
    *reinterpret_cast<float4*>(Es + row * B + c) = make_float4(s4[0], s4[1], s4[2], s4[3]);
    *reinterpret_cast<uint32_t*>(codes + row * cols + b0 + c) =
        static_cast<uint32_t>(qf[4 * t]) | (static_cast<uint32_t>(qf[4 * t + 1]) << 8) |
        (static_cast<uint32_t>(qf[4 * t + 2]) << 16) | (static_cast<uint32_t>(qf[4 * t + 3]) << 24);
  }
  if (sub == 0 && err_sq != nullptr) err_sq[row] += sq;
}

// Workspace: the tf32 split of E (rows x block, twice) and of the current block's rows of R
// (block x cols, twice).
size_t quantize_workspace_bytes(int64_t rows, int64_t cols, int block) {
  return 2 * align_up(static_cast<size_t>(rows) * block * 4, 256) +
         2 * align_up(static_cast<size_t>(block) * cols * 4, 256);
}

template <int B>
static gptq_status launch_column_loop(float* Wh, int64_t rows, int64_t cols, const float* R, int b0,
                                      int nb, int bits, int group, int group_mode, int gi_fixed,
                                      float* scales, uint8_t* zeros, int G, uint8_t* codes,
                                      float* Eb, float* Es, float* err_sq, float* Rb, float* Rs,
                                      int64_t nrest, int32_t* info, cudaStream_t stream) {
  // TPR lanes per row, 128 / TPR rows per CTA
  constexpr int TPR = 8, THREADS = 128, ROWS_PER_CTA = THREADS / TPR;
  const int64_t grid = (rows + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  constexpr int smem = (B * B + B) * 4;
  auto kernel = group_mode == 1 ? column_loop_kernel<B, 1, TPR> : column_loop_kernel<B, 0, TPR>;
  const gptq_status st = set_max_dynamic_smem(reinterpret_cast<const void*>(kernel), smem);
  if (st != GPTQ_OK) return st;
  return launch_pdl(kernel, dim3(static_cast<unsigned>(grid)), dim3(THREADS), smem, stream, Wh,
                    rows, cols, R, b0, nb, bits, group, gi_fixed, scales, zeros, G, codes, Eb, Es,
                    err_sq, Rb, Rs, nrest, info);
}

gptq_status run_quantize_layer(const void* W, gptq_dtype w_dtype, int64_t rows, int64_t cols,
                               int64_t ldw, const float* R, int bits, int group, int block,
                               float* Wh, uint8_t* codes, float* scales, uint8_t* zeros,
                               float* err_sq, void* ws, int32_t* info, cudaStream_t stream) {
  uint8_t* wp = static_cast<uint8_t*>(ws);
  const size_t e_bytes = align_up(static_cast<size_t>(rows) * block * 4, 256);
  const size_t r_bytes = align_up(static_cast<size_t>(block) * cols * 4, 256);
  float* Eb = reinterpret_cast<float*>(wp);
  float* Es = reinterpret_cast<float*>(wp + e_bytes);
  float* Rb = reinterpret_cast<float*>(wp + 2 * e_bytes);
  float* Rs = reinterpret_cast<float*>(wp + 2 * e_bytes + r_bytes);
  const int G = group > 0 ? static_cast<int>(cols / group) : 1;
  const int64_t total = rows * cols;
  const int cgrid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 8 * 148));
  if (w_dtype == GPTQ_BF16 && cols % 8 == 0 && ldw % 8 == 0 &&
      (reinterpret_cast<uintptr_t>(W) & 15) == 0)
    GPTQ_TRY_Q(launch_pdl(convert_bf16_vec_kernel,
                          dim3(static_cast<unsigned>(std::min<int64_t>((total / 8 + 255) / 256,
                                                                       8 * 148))),
                          dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(W), ldw, Wh, rows,
                          cols));
  else if (w_dtype == GPTQ_BF16)
    GPTQ_TRY_Q(launch_pdl(convert_kernel<__nv_bfloat16>, dim3(cgrid), dim3(256), 0, stream,
                          static_cast<const __nv_bfloat16*>(W), ldw, Wh, rows, cols));
  else
    GPTQ_TRY_Q(launch_pdl(convert_kernel<float>, dim3(cgrid), dim3(256), 0, stream,
                          static_cast<const float*>(W), ldw, Wh, rows, cols));
  if (err_sq != nullptr && cudaMemsetAsync(err_sq, 0, rows * sizeof(float), stream) != cudaSuccess)
    return GPTQ_ECUDA;
  const unsigned pgrid = static_cast<unsigned>((rows + 7) / 8);
  if (group <= 0) {
    GPTQ_TRY_Q(launch_pdl(params_kernel, dim3(pgrid), dim3(256), 0, stream, Wh, rows, cols, 0, cols,
                          bits, scales, zeros, 1, 0));
  }
  for (int64_t b0 = 0; b0 < cols; b0 += block) {
    const int nb = static_cast<int>(cols - b0 < block ? cols - b0 : block);
    int mode = 0, gi = 0;
    const int64_t b1 = b0 + nb, nrest = cols - b1;
    if (group > 0 && group % block == 0 && group != block) {
      gi = static_cast<int>(b0 / group);
      if (b0 % group == 0) {
        GPTQ_TRY_Q(launch_pdl(params_kernel, dim3(pgrid), dim3(256), 0, stream, Wh, rows, cols, b0,
                              static_cast<int64_t>(group), bits, scales, zeros, G, gi));
      }
    } else if (group > 0) {
      mode = 1;
    }
    // the column loop also writes the tf32 split of R[b0:b1, b1:] into (Rb, Rs) for S8
    gptq_status st;
    switch (block) {
      case 32:
        st = launch_column_loop<32>(Wh, rows, cols, R, static_cast<int>(b0), nb, bits, group, mode,
                                    gi, scales, zeros, G, codes, Eb, Es, err_sq, Rb, Rs, nrest,
                                    info, stream);
        break;
      case 64:
        st = launch_column_loop<64>(Wh, rows, cols, R, static_cast<int>(b0), nb, bits, group, mode,
                                    gi, scales, zeros, G, codes, Eb, Es, err_sq, Rb, Rs, nrest,
                                    info, stream);
        break;
      default:
        st = launch_column_loop<128>(Wh, rows, cols, R, static_cast<int>(b0), nb, bits, group,
                                     mode, gi, scales, zeros, G, codes, Eb, Es, err_sq, Rb, Rs,
                                     nrest, info, stream);
        break;
    }
    if (st != GPTQ_OK) return st;
    if (b1 < cols) {
      // S8: W[:, b1:] -= E * R[b0:b1, b1:] on the tensor cores (3xTF32)
      TcGemmArgs g{Eb, Es, Rb + b1, Rs + b1, block, cols, 0, 1,
                   static_cast<int>(rows), static_cast<int>(nrest), nb, -1.f, 1.f, 0, 0, 0,
                   Wh + b1, cols, nullptr, nullptr, 0, info};
      st = launch_gemm_tc(g, stream);
      if (st != GPTQ_OK) return st;
    }
  }
  return GPTQ_OK;
}

}  // namespace gptq
