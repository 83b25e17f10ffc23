// fp32-accurate matrix products on the tcgen05 tensor cores ("3xTF32").
//
// Every operand x is stored twice: x_big = x rounded to tf32 (10 explicit mantissa bits) and
// x_small = x - x_big (exact in fp32). The product is a_big*b_big + (a_big*b_small + a_small*b_big);
// the dropped a_small*b_small term and the tf32 truncation of the small parts leave a relative
// error near 2^-21 per product, close to fp32.
//
// The tensor core adds each MMA's result into its fp32 accumulator with a rounding biased toward
// zero, so long sums drift. The kernel therefore keeps two short-lived TMEM accumulators (the
// big*big term and the two correction terms) per chunk of kChunkStages k-stages and folds each
// chunk into a per-thread fp32 register accumulator with ordinary IEEE adds; the chunk buffers are
// double-buffered so the MMAs never wait for the fold.
//
// One CTA per 128 x 128 output tile: warp 0 issues TMA loads (128-byte swizzle, either operand
// K-major or MN-major), warp 1 issues the MMAs, warps 2-5 fold and write the tile:
//   C = alpha * acc + beta * C    (C may be null), and optionally the tf32 split of the result.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace tg {
constexpr int BM = 128, BN = 128, BK = 32;
constexpr int kStages = 3;
constexpr int kChunkStages = 8;                 // k-stages (256 k) per TMEM chunk sum
constexpr int kOpBytes = BM * BK * 4;           // 16 KB per operand part per stage
constexpr int kStageBytes = 4 * kOpBytes;       // A_big, A_small, B_big, B_small
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;             // 2 buffers x (main 128 + corr 128)
}  // namespace tg

__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

struct TcGemmParams {
  int M, N, K;
  int a_mn, b_mn;          // operand is MN-major (1) or K-major (0)
  float alpha, beta;
  int lower, klo_from_m, klo_from_n;
  float* C;                // may be null
  int64_t ldc;
  float* Cbig;             // may be null: tf32 split of the result
  float* Csmall;
  int64_t ld_split;
  int tiles_n;
  int vec4;                // C / split rows are 16-byte aligned
  int tiles_m, n_tiles;    // used by the persistent K <= 128 variant
  int stage_c;             // K <= 128 variant: C goes through shared memory by TMA
  int khi_from_m;
  int bstride;             // diagonal shift between batches (elements)
};

// tile index -> (tm, tn): row-major over all tiles, or over the lower triangle tn <= tm
__device__ __forceinline__ void tile_coords(const TcGemmParams& p, int t, int& tm, int& tn) {
  if (p.lower) {
    int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
    while ((i + 1) * (i + 2) / 2 <= t) ++i;
    while (i * (i + 1) / 2 > t) --i;
    tm = i;
    tn = t - i * (i + 1) / 2;
  } else {
    tm = t / p.tiles_n;
    tn = t - tm * p.tiles_n;
  }
}

__global__ void __launch_bounds__(tg::kThreads, 1)
gemm_tf32x3_tc(const __grid_constant__ CUtensorMap tAb, const __grid_constant__ CUtensorMap tAs,
               const __grid_constant__ CUtensorMap tBb, const __grid_constant__ CUtensorMap tBs,
               TcGemmParams p, int32_t* info) {
  using namespace tg;
  const int per_batch = p.tiles_m * p.tiles_n;
  const int bt = blockIdx.x / per_batch;
  // With k stopping after the tile's rows the later row tiles are the longer ones: they take the
  // first CTAs, so the last wave is made of the short tiles (longest first).
  const int tix0 = blockIdx.x - bt * per_batch;
  const int tix = p.khi_from_m ? per_batch - 1 - tix0 : tix0;
  const int tm = tix / p.tiles_n, tn = tix - (tix / p.tiles_n) * p.tiles_n;
  const int m0 = tm * BM, n0 = tn * BN;
  const int boff = bt * p.bstride;          // this batch's shift along the diagonal
  if (p.lower && n0 > m0 + BM - 1) return;  // tile entirely above the diagonal
  int klo = 0;
  if (p.klo_from_m) klo = max(klo, m0);
  if (p.klo_from_n) klo = max(klo, n0);
  const int khi = p.khi_from_m ? min(p.K, m0 + BM) : p.K;
  const int nk = khi > klo ? (khi - klo + BK - 1) / BK : 0;
  const int n_chunks = (nk + kChunkStages - 1) / kChunkStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  griddep_wait();                       // the previous kernel's results are visible from here
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0 && nk > 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, info)) break;
        uint8_t* st = smem + s * kStageBytes;
        const int k0 = klo + kb * BK + boff;
        const int am = m0 + boff, bn = n0 + boff;
        mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
        // A parts at st + 0 / kOpBytes, B parts at st + 2 / 3 * kOpBytes
        if (p.a_mn) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tma_load_2d(st + q * 4096, &tAb, &full_bar[s], am + 32 * q, k0);
            tma_load_2d(st + kOpBytes + q * 4096, &tAs, &full_bar[s], am + 32 * q, k0);
          }
        } else {
          tma_load_2d(st, &tAb, &full_bar[s], k0, am);
          tma_load_2d(st + kOpBytes, &tAs, &full_bar[s], k0, am);
        }
        if (p.b_mn) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tma_load_2d(st + 2 * kOpBytes + q * 4096, &tBb, &full_bar[s], bn + 32 * q, k0);
            tma_load_2d(st + 3 * kOpBytes + q * 4096, &tBs, &full_bar[s], bn + 32 * q, k0);
          }
        } else {
          tma_load_2d(st + 2 * kOpBytes, &tBb, &full_bar[s], k0, bn);
          tma_load_2d(st + 3 * kOpBytes, &tBs, &full_bar[s], k0, bn);
        }
        ++issued;
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0 && nk > 0) {
      const uint32_t idesc = make_idesc(/*tf32*/ 2, p.a_mn, p.b_mn, BM, BN);
      // K-major (128-byte swizzle): rows of 128 B in 8-row atoms; a K step of 8 tf32 is +32 B
      // inside the row. MN-major 32-bit operands must use the 128-byte swizzle with 32-byte atoms
      // (layout type 1): 128-byte rows in 4-row groups (SBO 512 B), 32-element MN chunks 4 KB
      // apart (LBO), a K step of 8 rows is +1024 B.
      const uint32_t a_lbo = p.a_mn ? 4096u : 16u, b_lbo = p.b_mn ? 4096u : 16u;
      const uint32_t a_sbo = p.a_mn ? 512u : 1024u, b_sbo = p.b_mn ? 512u : 1024u;
      const uint32_t a_lay = p.a_mn ? kSwizzle128B32BAtom : kSwizzle128B;
      const uint32_t b_lay = p.b_mn ? kSwizzle128B32BAtom : kSwizzle128B;
      const uint32_t a_step = p.a_mn ? 1024u : 32u, b_step = p.b_mn ? 1024u : 32u;
      int s = 0;
      uint32_t ph = 0;
      int kb = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int buf = c & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ((c >> 1) & 1) ^ 1u, &abort_flag, info)) break;
        tc_fence_after();
        const uint32_t t_main = tmem + buf * 256, t_corr = t_main + 128;
        const int kb_end = min(nk, kb + kChunkStages);
        bool first = true;
        bool ok = true;
        for (; kb < kb_end; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            const uint64_t ab = smem_desc(base + kk * a_step, a_lbo, a_sbo, a_lay);
            const uint64_t as = smem_desc(base + kOpBytes + kk * a_step, a_lbo, a_sbo, a_lay);
            const uint64_t bb = smem_desc(base + 2 * kOpBytes + kk * b_step, b_lbo, b_sbo, b_lay);
            const uint64_t bs = smem_desc(base + 3 * kOpBytes + kk * b_step, b_lbo, b_sbo, b_lay);
            tc_mma_tf32(t_corr, ab, bs, idesc, first ? 0u : 1u);
            tc_mma_tf32(t_corr, as, bb, idesc, 1u);
            tc_mma_tf32(t_main, ab, bb, idesc, first ? 0u : 1u);
            first = false;
          }
          tc_commit(&empty_bar[s]);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
      tc_commit(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else {
    // ---------------- epilogue: fold chunks into registers, then write ----------------
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    float acc[BN];
#pragma unroll
    for (int j = 0; j < BN; ++j) acc[j] = 0.f;
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int buf = c & 1;
      if (!mbar_wait_bounded(&acc_full[buf], (c >> 1) & 1, &abort_flag, info)) { ok = false; break; }
      tc_fence_after();
      const uint32_t t_main = tmem + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t vm[32], vc[32];
        tmem_ld_32x32b_x32(t_main + cc * 32, vm);
        tmem_ld_32x32b_x32(t_main + 128 + cc * 32, vc);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t)
          acc[cc * 32 + t] += __uint_as_float(vm[t]) + __uint_as_float(vc[t]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    if (ok && row < p.M) {
      const int64_t grow = row + boff, gcol = n0 + boff;
      float* crow = p.C ? p.C + grow * p.ldc + gcol : nullptr;
      float* brow = p.Cbig ? p.Cbig + grow * p.ld_split + gcol : nullptr;
      float* srow = p.Cbig ? p.Csmall + grow * p.ld_split + gcol : nullptr;
      const int ncol = min(BN, p.N - n0);
      if (p.vec4 && ncol == BN) {
#pragma unroll
        for (int j = 0; j < BN; j += 4) {
          float4 v = make_float4(p.alpha * acc[j], p.alpha * acc[j + 1], p.alpha * acc[j + 2],
                                 p.alpha * acc[j + 3]);
          if (p.beta != 0.f) {
            const float4 o = *reinterpret_cast<const float4*>(crow + j);
            v.x = fmaf(p.beta, o.x, v.x); v.y = fmaf(p.beta, o.y, v.y);
            v.z = fmaf(p.beta, o.z, v.z); v.w = fmaf(p.beta, o.w, v.w);
          }
          if (crow) *reinterpret_cast<float4*>(crow + j) = v;
          if (brow) {
            const float4 b = make_float4(tf32_round(v.x), tf32_round(v.y), tf32_round(v.z),
                                         tf32_round(v.w));
            *reinterpret_cast<float4*>(brow + j) = b;
            *reinterpret_cast<float4*>(srow + j) =
                make_float4(v.x - b.x, v.y - b.y, v.z - b.z, v.w - b.w);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < BN; ++j) {
          if (j < ncol) {
            float v = p.alpha * acc[j];
            if (p.beta != 0.f) v = fmaf(p.beta, crow[j], v);
            if (crow) crow[j] = v;
            if (brow) {
              const float b = tf32_round(v);
              brow[j] = b;
              srow[j] = v - b;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// K <= 128 products (the lazy trailing update, the Cholesky panel solve and trailing update, the
// triangular inverse's second product): persistent over a contiguous range of output tiles, A and
// B streamed through two 64 KB stages, two TMEM buffers so one tile's epilogue overlaps the next
// tile's MMAs.
//
// When C is 16-byte addressable the C tile goes through shared memory: four 128-row x 32-column
// boxes (128-byte swizzle) that one epilogue thread loads by TMA for the next tile as soon as the
// current tile's store of that box has left shared memory, so the epilogue never waits on a global
// load; the updated box is written back to shared memory (conflict-free, the swizzle spreads a
// warp's rows over all banks) and stored by TMA. The tf32 split of the result, when requested, is
// written straight from registers.
// ------------------------------------------------------------------------------------------------
namespace tgp {
constexpr int BM = 128, BN = 128, BK = 32;
constexpr int kMaxK = 128;
constexpr int kPartBytes = BM * BK * 4;             // 16 KB: one part (big or small) of one operand
constexpr int kStages = 2;
constexpr int kStageBytes = 4 * kPartBytes;         // A_big, A_small, B_big, B_small
constexpr int kBoxBytes = BM * 32 * 4;              // 16 KB: 128 rows x 32 columns of C
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kSmemBytesStaged = kSmemBytes + 4 * kBoxBytes;
constexpr int kThreads = 224;                       // warps: 0 A/B loads, 1 MMA, 2-5 epilogue, 6 C
constexpr int kIssuerWarp = 6;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kEpiBarrier = 1;                 // named barrier of the 128 epilogue threads
}  // namespace tgp

__global__ void __launch_bounds__(tgp::kThreads, 1)
gemm_tf32x3_panel_tc(const __grid_constant__ CUtensorMap tAb, const __grid_constant__ CUtensorMap tAs,
                     const __grid_constant__ CUtensorMap tBb, const __grid_constant__ CUtensorMap tBs,
                     const __grid_constant__ CUtensorMap tC, TcGemmParams p, int32_t* info) {
  using namespace tgp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ __align__(8) uint64_t cbox[4];        // box j may be written (and holds C if beta != 0)
  __shared__ __align__(8) uint64_t ready[4];       // box j written by the epilogue, may be stored
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.K + BK - 1) / BK;   // 1..4
  const int t_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.n_tiles / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.n_tiles / gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    for (int j = 0; j < 4; ++j) {
      mbar_init(&cbox[j], 1);
      mbar_init(&ready[j], 128);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  griddep_wait();                       // the previous kernel's results are visible from here
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      for (int t = t_begin; t < t_end && !abort_flag; ++t) {
        int tm, tn;
        tile_coords(p, t, tm, tn);
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, info)) goto producer_done;
          uint8_t* st = smem + s * kStageBytes;
          const int k0 = kb * BK;
          mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
          if (p.a_mn) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              tma_load_2d(st + q * 4096, &tAb, &full_bar[s], m0 + 32 * q, k0);
              tma_load_2d(st + kPartBytes + q * 4096, &tAs, &full_bar[s], m0 + 32 * q, k0);
            }
          } else {
            tma_load_2d(st, &tAb, &full_bar[s], k0, m0);
            tma_load_2d(st + kPartBytes, &tAs, &full_bar[s], k0, m0);
          }
          if (p.b_mn) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              tma_load_2d(st + 2 * kPartBytes + q * 4096, &tBb, &full_bar[s], n0 + 32 * q, k0);
              tma_load_2d(st + 3 * kPartBytes + q * 4096, &tBs, &full_bar[s], n0 + 32 * q, k0);
            }
          } else {
            tma_load_2d(st + 2 * kPartBytes, &tBb, &full_bar[s], k0, n0);
            tma_load_2d(st + 3 * kPartBytes, &tBs, &full_bar[s], k0, n0);
          }
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    producer_done:
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(/*tf32*/ 2, p.a_mn, p.b_mn, BM, BN);
      const uint32_t a_lbo = p.a_mn ? 4096u : 16u, b_lbo = p.b_mn ? 4096u : 16u;
      const uint32_t a_sbo = p.a_mn ? 512u : 1024u, b_sbo = p.b_mn ? 512u : 1024u;
      const uint32_t a_lay = p.a_mn ? kSwizzle128B32BAtom : kSwizzle128B;
      const uint32_t b_lay = p.b_mn ? kSwizzle128B32BAtom : kSwizzle128B;
      const uint32_t a_step = p.a_mn ? 1024u : 32u, b_step = p.b_mn ? 1024u : 32u;
      int s = 0, c = 0;
      uint32_t ph = 0;
      for (int t = t_begin; t < t_end && !abort_flag; ++t, ++c) {
        const int buf = c & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ((c >> 1) & 1) ^ 1u, &abort_flag, info))
          goto mma_done_label;
        tc_fence_after();
        const uint32_t t_main = tmem + buf * 256, t_corr = t_main + 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) goto mma_done_label;
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            const uint64_t ab = smem_desc(base + kk * a_step, a_lbo, a_sbo, a_lay);
            const uint64_t as = smem_desc(base + kPartBytes + kk * a_step, a_lbo, a_sbo, a_lay);
            const uint64_t bb = smem_desc(base + 2 * kPartBytes + kk * b_step, b_lbo, b_sbo, b_lay);
            const uint64_t bs = smem_desc(base + 3 * kPartBytes + kk * b_step, b_lbo, b_sbo, b_lay);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            tc_mma_tf32(t_corr, ab, bs, idesc, accum);
            tc_mma_tf32(t_corr, as, bb, idesc, 1u);
            tc_mma_tf32(t_main, ab, bb, idesc, accum);
          }
          tc_commit(&empty_bar[s]);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        tc_commit(&acc_full[buf]);
      }
    mma_done_label:
      tc_commit(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else if (warp == kIssuerWarp) {
    if (lane == 0 && p.stage_c) {
      // ---- C issuer: TMA stores of the boxes the epilogue finished, TMA loads of the next
      // tile's C into each box as soon as its store has left shared memory ----
      const bool loads = p.beta != 0.f;
      uint8_t* cs = smem + kStages * kStageBytes;
      uint32_t rdy_ph = 0;      // per-box parity of the next ready[] completion
      uint32_t rel = 0;         // boxes released at least once
      uint32_t last_ph = 0;     // per-box parity of the latest release's cbox completion
      auto release = [&](int m0n, int n0n, int j) {
        if (rel & (1u << j)) last_ph ^= 1u << j;
        rel |= 1u << j;
        if (loads) {
          mbar_arrive_expect_tx(&cbox[j], kBoxBytes);
          tma_load_2d(cs + j * kBoxBytes, &tC, &cbox[j], n0n + 32 * j, m0n);
        } else {
          mbar_arrive(&cbox[j]);
        }
      };
      auto n_boxes = [&](int n0) { return min(4, (p.N - n0 + 31) / 32); };
      if (t_begin < t_end) {
        int tm, tn;
        tile_coords(p, t_begin, tm, tn);
        const int nb0 = n_boxes(tn * BN);
        for (int j = 0; j < nb0; ++j) release(tm * BM, tn * BN, j);
      }
      for (int t = t_begin; t < t_end; ++t) {
        int tm, tn;
        tile_coords(p, t, tm, tn);
        const int m0 = tm * BM, n0 = tn * BN;
        const int nbx = n_boxes(n0);
        int nm0 = 0, nn0 = 0, nnb = 0;               // the next tile (nnb = 0: none)
        if (t + 1 < t_end) {
          int tm2, tn2;
          tile_coords(p, t + 1, tm2, tn2);
          nm0 = tm2 * BM;
          nn0 = tn2 * BN;
          nnb = n_boxes(nn0);
        }
        bool ok = true;
        for (int j = 0; j < nbx; ++j) {
          if (!mbar_wait_bounded(&ready[j], (rdy_ph >> j) & 1u, &abort_flag, info)) {
            ok = false;
            break;
          }
          rdy_ph ^= 1u << j;
          tma_store_2d(&tC, cs + j * kBoxBytes, n0 + 32 * j, m0);
          tma_store_commit();
          if (j >= 1) {
            tma_store_wait_read<1>();                // box j-1 has left shared memory
            if (j - 1 < nnb) release(nm0, nn0, j - 1);
          }
        }
        if (!ok) break;
        tma_store_wait_read<0>();
        for (int j = nbx - 1; j < nnb; ++j) release(nm0, nn0, j);
      }
      tma_store_wait_all();
      if (loads)
        for (int j = 0; j < 4; ++j)
          if (rel & (1u << j)) mbar_drain_bounded(&cbox[j], (last_ph >> j) & 1u);
    }
  } else if (p.stage_c) {
    // ---- epilogue through shared memory: fold TMEM, write the four 128 x 32 boxes (swizzled),
    // hand each to the C issuer ----
    const int q = warp & 3;
    const int r = q * 32 + lane;                    // row within the tile (= TMEM lane)
    const int et = threadIdx.x - 64;                // 0..127 within the epilogue group
    const uint32_t rsw = static_cast<uint32_t>(r & 7);
    const bool loads = p.beta != 0.f;
    const bool split = p.Cbig != nullptr;
    uint8_t* cs = smem + kStages * kStageBytes;
    uint32_t tok_ph = 0;                            // per-box parity of the next cbox completion
    auto n_boxes = [&](int n0) { return min(4, (p.N - n0 + 31) / 32); };
    int c = 0;
    for (int t = t_begin; t < t_end; ++t, ++c) {
      int tm, tn;
      tile_coords(p, t, tm, tn);
      const int m0 = tm * BM, n0 = tn * BN;
      const int nbx = n_boxes(n0);
      const int buf = c & 1;
      const bool ok = mbar_wait_bounded(&acc_full[buf], (c >> 1) & 1, &abort_flag, info);
      if (named_barrier_or(kEpiBarrier, 128, !ok || abort_flag)) break;
      tc_fence_after();
      float acc[BN];
      const uint32_t t_main = tmem + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t vm[32], vc[32];
        tmem_ld_32x32b_x32(t_main + cc * 32, vm);
        tmem_ld_32x32b_x32(t_main + 128 + cc * 32, vc);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) acc[cc * 32 + u] = __uint_as_float(vm[u]) + __uint_as_float(vc[u]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      bool stop = false;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j < nbx) {
          bool okc = !stop && mbar_wait_bounded(&cbox[j], (tok_ph >> j) & 1u, &abort_flag, info);
          uint8_t* box = cs + j * kBoxBytes;
          if (okc) {
            tok_ph ^= 1u << j;
            uint8_t* rowp = box + r * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              float4* a = reinterpret_cast<float4*>(rowp + ((static_cast<uint32_t>(u) ^ rsw) << 4));
              const float* x = acc + j * 32 + 4 * u;
              float4 v = make_float4(p.alpha * x[0], p.alpha * x[1], p.alpha * x[2], p.alpha * x[3]);
              if (loads) {
                const float4 o = *a;
                v.x = fmaf(p.beta, o.x, v.x); v.y = fmaf(p.beta, o.y, v.y);
                v.z = fmaf(p.beta, o.z, v.z); v.w = fmaf(p.beta, o.w, v.w);
              }
              *a = v;
            }
          }
          stop = !okc;
          if (split) {
            // the tf32 split of the box, written row-contiguous from shared memory
            stop = named_barrier_or(kEpiBarrier, 128, stop || abort_flag);
            if (!stop) {
#pragma unroll
              for (int s2 = 0; s2 < 8; ++s2) {
                const int f = et + 128 * s2;
                const int br = f >> 3, u = f & 7;
                const float4 v = *reinterpret_cast<const float4*>(
                    box + br * 128 + ((static_cast<uint32_t>(u) ^ static_cast<uint32_t>(br & 7)) << 4));
                const int row = m0 + br, col = n0 + 32 * j + 4 * u;
                if (row < p.M) {
                  const float4 bg = make_float4(tf32_round(v.x), tf32_round(v.y), tf32_round(v.z),
                                                tf32_round(v.w));
                  const float4 sm = make_float4(v.x - bg.x, v.y - bg.y, v.z - bg.z, v.w - bg.w);
                  float* bp = p.Cbig + static_cast<int64_t>(row) * p.ld_split + col;
                  float* sp = p.Csmall + static_cast<int64_t>(row) * p.ld_split + col;
                  if (col + 4 <= p.N) {
                    *reinterpret_cast<float4*>(bp) = bg;
                    *reinterpret_cast<float4*>(sp) = sm;
                  } else {
                    const float bb[4] = {bg.x, bg.y, bg.z, bg.w}, ss[4] = {sm.x, sm.y, sm.z, sm.w};
                    for (int e = 0; e < 4 && col + e < p.N; ++e) {
                      bp[e] = bb[e];
                      sp[e] = ss[e];
                    }
                  }
                }
              }
            }
          }
          if (!stop) {
            fence_proxy_async_smem();
            mbar_arrive(&ready[j]);
          }
        }
      }
    }
  } else {
    const int q = warp & 3;
    int c = 0;
    for (int t = t_begin; t < t_end && !abort_flag; ++t, ++c) {
      int tm, tn;
      tile_coords(p, t, tm, tn);
      const int m0 = tm * BM, n0 = tn * BN;
      const int buf = c & 1;
      if (!mbar_wait_bounded(&acc_full[buf], (c >> 1) & 1, &abort_flag, info)) break;
      tc_fence_after();
      float acc[BN];
      const uint32_t t_main = tmem + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t vm[32], vc[32];
        tmem_ld_32x32b_x32(t_main + cc * 32, vm);
        tmem_ld_32x32b_x32(t_main + 128 + cc * 32, vc);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) acc[cc * 32 + u] = __uint_as_float(vm[u]) + __uint_as_float(vc[u]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);   // the buffer is free as soon as the sums are in registers
      const int row = m0 + q * 32 + lane;
      if (row < p.M) {
        float* crow = p.C ? p.C + static_cast<int64_t>(row) * p.ldc + n0 : nullptr;
        float* brow = p.Cbig ? p.Cbig + static_cast<int64_t>(row) * p.ld_split + n0 : nullptr;
        float* srow = p.Cbig ? p.Csmall + static_cast<int64_t>(row) * p.ld_split + n0 : nullptr;
        const int ncol = min(BN, p.N - n0);
        if (p.vec4 && ncol == BN) {
#pragma unroll
          for (int j = 0; j < BN; j += 4) {
            float4 v = make_float4(p.alpha * acc[j], p.alpha * acc[j + 1], p.alpha * acc[j + 2],
                                   p.alpha * acc[j + 3]);
            if (p.beta != 0.f) {
              const float4 o = *reinterpret_cast<const float4*>(crow + j);
              v.x = fmaf(p.beta, o.x, v.x); v.y = fmaf(p.beta, o.y, v.y);
              v.z = fmaf(p.beta, o.z, v.z); v.w = fmaf(p.beta, o.w, v.w);
            }
            if (crow) *reinterpret_cast<float4*>(crow + j) = v;
            if (brow) {
              const float4 b = make_float4(tf32_round(v.x), tf32_round(v.y), tf32_round(v.z),
                                           tf32_round(v.w));
              *reinterpret_cast<float4*>(brow + j) = b;
              *reinterpret_cast<float4*>(srow + j) =
                  make_float4(v.x - b.x, v.y - b.y, v.z - b.z, v.w - b.w);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            if (j < ncol) {
              float v = p.alpha * acc[j];
              if (p.beta != 0.f) v = fmaf(p.beta, crow[j], v);
              if (crow) crow[j] = v;
              if (brow) {
                const float b = tf32_round(v);
                brow[j] = b;
                srow[j] = v - b;
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// The lazy trailing update's shape (S8: C += alpha * A B with A K-major, B MN-major, K <= 128,
// whole 128-column tiles, beta = 1): the same product with the A row band kept in shared memory.
// A CTA's tiles are consecutive in row-major order, so most of them share their A band; the band
// (up to 4 k-blocks x big/small = 128 KB) is loaded once per band and only B is streamed (two
// 32 KB stages), which halves the operand bytes per tile. C is never read by the CTA: each
// 128 x 32 box of alpha * acc goes into one of two shared buffers and a TMA reduce-add adds it
// into C in L2 (one fp32 add per element, the same rounding as reading C and adding).
// ------------------------------------------------------------------------------------------------
namespace tga {
constexpr int BM = 128, BN = 128, BK = 32, kMaxKb = 4;
constexpr int kPartBytes = BM * BK * 4;                 // 16 KB: one part (big or small)
constexpr int kABytes = kMaxKb * 2 * kPartBytes;        // the A band: k-block kb at kb * 32 KB
constexpr int kStages = 2;
constexpr int kStageBytes = 2 * kPartBytes;             // B_big, B_small
constexpr int kBoxBytes = BM * 32 * 4;                  // 16 KB
constexpr int kBoxes = 2;
constexpr int kSmemBytes = kABytes + kStages * kStageBytes + kBoxes * kBoxBytes + 1024;
constexpr int kThreads = 224;                           // 0 loads, 1 MMA, 2-5 epilogue, 6 C
constexpr int kIssuerWarp = 6;
constexpr uint32_t kTmemCols = 512;
}  // namespace tga

__global__ void __launch_bounds__(tga::kThreads, 1)
gemm_tf32x3_aband_tc(const __grid_constant__ CUtensorMap tAb, const __grid_constant__ CUtensorMap tAs,
                     const __grid_constant__ CUtensorMap tBb, const __grid_constant__ CUtensorMap tBs,
                     const __grid_constant__ CUtensorMap tC, TcGemmParams p, int32_t* info) {
  using namespace tga;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  uint8_t* sa = smem;                                   // the A band
  uint8_t* sb = smem + kABytes;                         // B stages
  uint8_t* cs = sb + kStages * kStageBytes;             // C boxes
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t a_full, a_empty;
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ __align__(8) uint64_t cbox[kBoxes];        // box b may be written
  __shared__ __align__(8) uint64_t ready[kBoxes];       // box b written by the epilogue
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.K + BK - 1) / BK;   // 1..4
  const int t_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.n_tiles / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.n_tiles / gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&a_full, 1);
    mbar_init(&a_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    for (int b = 0; b < kBoxes; ++b) {
      mbar_init(&cbox[b], 1);
      mbar_init(&ready[b], 128);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ---------------- loads: the A band when it changes, B per tile ----------------
    if (lane == 0) {
      int s = 0, issued = 0, bands = 0, band = -1;
      uint32_t ph = 0;
      for (int t = t_begin; t < t_end && !abort_flag; ++t) {
        const int tm = t / p.tiles_n, tn = t - tm * p.tiles_n;
        const int m0 = tm * BM, n0 = tn * BN;
        if (tm != band) {
          // the MMAs of the previous band are done with it
          if (bands > 0 &&
              !mbar_wait_bounded(&a_empty, static_cast<uint32_t>((bands - 1) & 1), &abort_flag, info))
            goto producer_done;
          mbar_arrive_expect_tx(&a_full, static_cast<uint32_t>(nk) * 2u * kPartBytes);
          for (int kb = 0; kb < nk; ++kb) {
            tma_load_2d(sa + kb * 2 * kPartBytes, &tAb, &a_full, kb * BK, m0);
            tma_load_2d(sa + kb * 2 * kPartBytes + kPartBytes, &tAs, &a_full, kb * BK, m0);
          }
          band = tm;
          ++bands;
        }
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, info)) goto producer_done;
          uint8_t* st = sb + s * kStageBytes;
          mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tma_load_2d(st + q * 4096, &tBb, &full_bar[s], n0 + 32 * q, kb * BK);
            tma_load_2d(st + kPartBytes + q * 4096, &tBs, &full_bar[s], n0 + 32 * q, kb * BK);
          }
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    producer_done:
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
      if (bands > 0) mbar_drain_bounded(&a_full, static_cast<uint32_t>((bands - 1) & 1));
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = make_idesc(/*tf32*/ 2, 0, 1, BM, BN);
      int s = 0, c = 0, bands = 0, band = -1;
      uint32_t ph = 0;
      for (int t = t_begin; t < t_end && !abort_flag; ++t, ++c) {
        const int tm = t / p.tiles_n;
        const int buf = c & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ((c >> 1) & 1) ^ 1u, &abort_flag, info))
          goto mma_finish;
        if (tm != band) {
          if (!mbar_wait_bounded(&a_full, static_cast<uint32_t>(bands & 1), &abort_flag, info))
            goto mma_finish;
          band = tm;
          ++bands;
        }
        tc_fence_after();
        const uint32_t t_main = tmem + buf * 256, t_corr = t_main + 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) goto mma_finish;
          tc_fence_after();
          const uint32_t abase = smem_u32(sa + kb * 2 * kPartBytes);
          const uint32_t bbase = smem_u32(sb + s * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            // A K-major (128-byte swizzle, +32 B per 8 k); B MN-major (128-byte swizzle with
            // 32-byte atoms: 32-element chunks 4 KB apart, +1024 B per 8 k)
            const uint64_t ab = smem_desc(abase + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t as = smem_desc(abase + kPartBytes + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bb = smem_desc(bbase + kk * 1024, 4096, 512, kSwizzle128B32BAtom);
            const uint64_t bs =
                smem_desc(bbase + kPartBytes + kk * 1024, 4096, 512, kSwizzle128B32BAtom);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            tc_mma_tf32(t_corr, ab, bs, idesc, accum);
            tc_mma_tf32(t_corr, as, bb, idesc, 1u);
            tc_mma_tf32(t_main, ab, bb, idesc, accum);
          }
          tc_commit(&empty_bar[s]);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        tc_commit(&acc_full[buf]);
        // the band is released once the last tile using it is done
        if (t + 1 == t_end || (t + 1) / p.tiles_n != tm) tc_commit(&a_empty);
      }
    mma_finish:
      tc_commit(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else if (warp == kIssuerWarp) {
    // ---------------- C boxes: a tile's four column boxes go through two buffers in turn, each
    // added into C by a TMA reduce-add and handed back once it has been read out ----------
    if (lane == 0) {
      uint32_t rdy_ph = 0;
      for (int b = 0; b < kBoxes; ++b) mbar_arrive(&cbox[b]);
      bool ok = true;
      for (int t = t_begin; ok && t < t_end; ++t) {
        const int tm = t / p.tiles_n, tn = t - tm * p.tiles_n;
        for (int j = 0; j < 4; ++j) {
          const int b = j & 1;
          if (!mbar_wait_bounded(&ready[b], (rdy_ph >> b) & 1u, &abort_flag, info)) {
            ok = false;
            break;
          }
          rdy_ph ^= 1u << b;
          tma_reduce_add_2d(&tC, cs + b * kBoxBytes, tn * BN + 32 * j, tm * BM);
          tma_store_commit();
          tma_store_wait_read<0>();           // the buffer has left shared memory
          mbar_arrive(&cbox[b]);
        }
      }
      tma_store_wait_all();
    }
  } else if (warp >= 2 && warp < 6) {
    // ---------------- epilogue: fold TMEM, alpha * acc into the boxes ----------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t rsw = static_cast<uint32_t>(r & 7);
    uint32_t tok_ph = 0;
    int c = 0;
    for (int t = t_begin; t < t_end; ++t, ++c) {
      const int buf = c & 1;
      const bool ok = mbar_wait_bounded(&acc_full[buf], (c >> 1) & 1, &abort_flag, info);
      if (named_barrier_or(1, 128, !ok || abort_flag)) break;
      tc_fence_after();
      float acc[BN];
      const uint32_t t_main = tmem + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t vm[32], vc[32];
        tmem_ld_32x32b_x32(t_main + cc * 32, vm);
        tmem_ld_32x32b_x32(t_main + 128 + cc * 32, vc);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) acc[cc * 32 + u] = __uint_as_float(vm[u]) + __uint_as_float(vc[u]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      bool stop = false;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int b = j & 1;
        const bool okc = !stop && mbar_wait_bounded(&cbox[b], (tok_ph >> b) & 1u, &abort_flag, info);
        if (okc) {
          tok_ph ^= 1u << b;
          uint8_t* rowp = cs + b * kBoxBytes + r * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float4* a = reinterpret_cast<float4*>(rowp + ((static_cast<uint32_t>(u) ^ rsw) << 4));
            const float* x = acc + j * 32 + 4 * u;
            *a = make_float4(p.alpha * x[0], p.alpha * x[1], p.alpha * x[2], p.alpha * x[3]);
          }
        }
        // every epilogue thread takes the same branch (a lost wait stops all of them)
        stop = named_barrier_or(1, 128, !okc || abort_flag);
        if (!stop) {
          fence_proxy_async_smem();
          mbar_arrive(&ready[b]);
        }
      }
      if (stop) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// x -> (tf32(x), x - tf32(x)) for a rows x cols block (row-major, leading dims in elements).
__global__ void split_tf32_kernel(const float* __restrict__ X, int64_t ldx, int64_t rows,
                                  int64_t cols, float* __restrict__ big, float* __restrict__ small,
                                  int64_t ldo) {
  griddep_wait();
  griddep_launch_dependents();

  const int64_t total = rows * cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    const float x = X[r * ldx + c];
    const float b = tf32_round(x);
    big[r * ldo + c] = b;
    small[r * ldo + c] = x - b;
  }
}

gptq_status launch_split_tf32(const float* X, int64_t ldx, int64_t rows, int64_t cols, float* big,
                              float* small, int64_t ldo, cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return GPTQ_OK;
  const int64_t total = rows * cols;
  const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 16 * 148));
  return launch_pdl(split_tf32_kernel, dim3(grid), dim3(256), 0, stream, X, ldx, rows, cols, big,
                    small, ldo);
}

static gptq_status operand_map(CUtensorMap* m, const float* base, int64_t ld, int mn_major,
                               int64_t mn_extent, int64_t k_extent) {
  // K-major: dims {K, MN}, box {32, 128}, 128-byte swizzle; MN-major: dims {MN, K}, box {32, 32},
  // 128-byte swizzle with 32-byte atoms (the only MN-major layout tcgen05 takes for tf32).
  if (mn_major)
    return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, 4, mn_extent, k_extent, ld,
                          32, 32, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, 4, k_extent, mn_extent, ld, 32,
                        128, CU_TENSOR_MAP_SWIZZLE_128B);
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gptq_status launch_gemm_tc(const TcGemmArgs& g, cudaStream_t stream) {
  using namespace tg;
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return GPTQ_OK;
  if (!al16(g.Ab) || !al16(g.As) || !al16(g.Bb) || !al16(g.Bs) || g.lda % 4 || g.ldb % 4)
    return GPTQ_EINVAL;
  if (g.batch > 1 && (g.bstride <= 0 || g.bstride % 4 || g.bstride > (1 << 24))) return GPTQ_EINVAL;
  const int K = g.K > 0 ? g.K : 1;  // an empty K still needs valid maps
  // the maps span every batch: batch b reads rows/columns shifted by b * bstride
  const int64_t ext = g.batch > 1 ? (g.batch - 1) * g.bstride : 0;
  CUtensorMap tAb, tAs, tBb, tBs;
  gptq_status st;
  if ((st = operand_map(&tAb, g.Ab, g.lda, g.a_mn, g.M + ext, K + ext)) != GPTQ_OK) return st;
  if ((st = operand_map(&tAs, g.As, g.lda, g.a_mn, g.M + ext, K + ext)) != GPTQ_OK) return st;
  if ((st = operand_map(&tBb, g.Bb, g.ldb, g.b_mn, g.N + ext, K + ext)) != GPTQ_OK) return st;
  if ((st = operand_map(&tBs, g.Bs, g.ldb, g.b_mn, g.N + ext, K + ext)) != GPTQ_OK) return st;
  if ((st = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_tf32x3_tc), kSmemBytes)) !=
      GPTQ_OK)
    return st;
  TcGemmParams p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.a_mn = g.a_mn; p.b_mn = g.b_mn;
  p.alpha = g.alpha; p.beta = g.beta;
  p.lower = g.lower; p.klo_from_m = g.klo_from_m; p.klo_from_n = g.klo_from_n;
  p.C = g.C; p.ldc = g.ldc;
  p.Cbig = g.Cbig; p.Csmall = g.Csmall; p.ld_split = g.ld_split;
  p.tiles_n = (g.N + BN - 1) / BN;
  const int tiles_m = (g.M + BM - 1) / BM;
  p.vec4 = ((g.C == nullptr || (al16(g.C) && g.ldc % 4 == 0)) &&
            (g.Cbig == nullptr || (al16(g.Cbig) && al16(g.Csmall) && g.ld_split % 4 == 0)))
               ? 1 : 0;
  p.tiles_m = tiles_m;
  p.stage_c = 0;
  p.khi_from_m = g.khi_from_m;
  p.bstride = static_cast<int>(g.batch > 1 ? g.bstride : 0);
  const bool panel = g.K > 0 && g.K <= tgp::kMaxK && !g.klo_from_m && !g.klo_from_n &&
                     !g.khi_from_m && g.batch == 1 && (!g.lower || g.M == g.N);
  if (panel) {
    if ((st = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_tf32x3_panel_tc),
                                   tgp::kSmemBytesStaged)) != GPTQ_OK)
      return st;
    const int64_t nt = g.lower ? static_cast<int64_t>(tiles_m) * (tiles_m + 1) / 2
                               : static_cast<int64_t>(tiles_m) * p.tiles_n;
    if (nt > 0x7fffffff) return GPTQ_EUNSUPPORTED;
    p.n_tiles = static_cast<int>(nt);
    // C through shared memory when a TMA map can describe it (16-byte base and row pitch)
    CUtensorMap tC;
    memset(&tC, 0, sizeof(tC));
    p.stage_c = (g.C != nullptr && p.vec4) ? 1 : 0;
    if (p.stage_c &&
        (st = encode_tmap_2d(&tC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.C, 4, g.N, g.M, g.ldc, 32,
                             tgp::BM, CU_TENSOR_MAP_SWIZZLE_128B)) != GPTQ_OK)
      return st;
    const int grid = p.n_tiles < num_sms() ? p.n_tiles : num_sms();
    if (p.stage_c && !g.a_mn && g.b_mn && !g.lower && g.Cbig == nullptr && g.beta == 1.f &&
        g.N % tga::BN == 0) {
      // the lazy trailing update's shape: the A band stays in shared memory
      if ((st = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_tf32x3_aband_tc),
                                     tga::kSmemBytes)) != GPTQ_OK)
        return st;
      return launch_pdl(gemm_tf32x3_aband_tc, dim3(grid), dim3(tga::kThreads), tga::kSmemBytes,
                        stream, tAb, tAs, tBb, tBs, tC, p, g.info);
    }
    const int smem = p.stage_c ? tgp::kSmemBytesStaged : tgp::kSmemBytes;
    return launch_pdl(gemm_tf32x3_panel_tc, dim3(grid), dim3(tgp::kThreads), smem, stream, tAb,
                      tAs, tBb, tBs, tC, p, g.info);
  } else {
    const int64_t grid = static_cast<int64_t>(tiles_m) * p.tiles_n * g.batch;
    if (grid > 0x7fffffff) return GPTQ_EUNSUPPORTED;
    p.n_tiles = static_cast<int>(grid);
    return launch_pdl(gemm_tf32x3_tc, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmemBytes,
                      stream, tAb, tAs, tBb, tBs, p, g.info);
  }
}

}  // namespace gptq
