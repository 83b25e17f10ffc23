// One fused step of the blocked right-looking Cholesky (S3/S5) on the tcgen05 tensor cores.
//
// "GPTQ second-order quantization" blog, "3. Cholesky reformulation"; "Part 3: Adaptive Rounding:
// GPTQ", "Algorithm GPTQ" (the Cholesky factor that the column loop reads).
//
// Step k of the factorization A = L L^T (128-wide blocks, T block rows) takes the inverse X_kk of
// the diagonal block L_kk (already factored) and in ONE launch does
//   P(i)   : the panel solve L_ik = A_ik X_kk^T for every block row i > k, and
//   U(i,j) : the trailing update A_ij -= L_ik L_jk^T for k < j <= i,
// and, on its first CTA, factors the next diagonal block A_{k+1,k+1} as soon as that block's own
// update is done, while the other CTAs are still busy with the rest of the trailing update. The
// chain from one diagonal block to the next is therefore one panel tile, one update tile and the
// on-chip factorization, with no launch in between and no wait for the whole trailing update.
//
// Every tile product is a K = 128 product in 3xTF32 (see gemm_tc.cu): operands as tf32 (big,
// small) pairs loaded by TMA, the big*big and correction terms in two TMEM accumulators.
//   P(i): A operand = the panel's split (written by the previous step's updates of block column
//         k, or by a split kernel for k = 0), B operand = X_kk's split. The result's split goes to
//         L's split (the later updates and the triangular inverse read it); L_ik itself goes to A
//         only when the caller keeps L there.
//   U(i,j): A operand = L_ik's split, B operand = L_jk's split, C = A_ij read and written through
//         shared memory by TMA. Tiles of block column k+1 (below the diagonal) also write the
//         split of the result: the next step's panel.
// An update tile waits for the panel tiles it reads on a per-block-row flag (the step number,
// stored with release semantics after the tile's split has been written; read with acquire
// semantics and a proxy fence before the TMA loads). Panel tiles wait on nothing and come first
// in every CTA's list, so every wait ends while all CTAs of the grid (at most one per SM) are
// resident; each wait is bounded in time all the same and reports GPTQ_INFO_TIMEOUT.
//
// CTA 0 computes P(k+1) for itself only: its epilogue writes the split straight from TMEM into the
// idle stage buffers, in the layout the MMA reads, and U(k+1, k+1) = A - L L^T multiplies that
// split by itself without a trip through global memory; the update lands in the diagonal block's
// shared layout (two warpgroups) and the factorization starts. CTA 1 computes the same P(k+1) as
// its first panel tile, for global memory and the flag, so CTA 0 never waits for a store.
//
// Warps: 0 loads A/B by TMA, 1 issues the MMAs, 2 moves C boxes by TMA, 4-7 fold TMEM and write
// (on CTA 0 also 8-11, for half of the diagonal block's update); all 16 run the diagonal block's
// factorization on CTA 0 afterwards.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "diag_block.cuh"
#include "internal.h"

namespace gptq {

namespace ps {
constexpr int BM = 128, BN = 128, BK = 32, NK = 4;    // K = 128: four k-stages per tile
constexpr int kPartBytes = BM * BK * 4;               // 16 KB: one part (big or small) of an operand
constexpr int kStages = 2;
constexpr int kStageBytes = 4 * kPartBytes;           // A_big, A_small, B_big, B_small
constexpr int kBoxBytes = BM * 32 * 4;                // 16 KB: 128 rows x 32 columns of C
constexpr int kBoxOffset = kStages * kStageBytes;
constexpr int kSmemBytes = kBoxOffset + 4 * kBoxBytes + 1024;
constexpr int kThreads = la::kDiagThreads;
constexpr int kMmaWarp = 1, kIssuerWarp = 2, kEpiWarp0 = 4;
constexpr uint32_t kEpiBar = 3;                       // named barrier of the 128 epilogue threads
constexpr uint32_t kEpiBar2 = 4;                      // CTA 0: warps 8-11 helping with one update
constexpr uint32_t kTmemCols = 512;                   // 2 buffers x (main 128 + correction 128)
static_assert(la::kDiagSmem + 1024 <= kSmemBytes, "the diagonal block must fit the tile buffers");
static_assert(la::kNB == BM, "one diagonal block per tile");
}  // namespace ps

struct StepParams {
  int n, T, k;
  int store_l, rev_n, info_base;
  int dx, dy;             // coordinates of X_kk's split in the tD maps
  int32_t* flags;         // [T]: flags[i] = s + 1 once L_is's split is written
  float* Lb;              // L's split (n x n, ld n)
  float* Ls;
  float* Pb[2];           // the panel split by parity of its step (n x 128 each, absolute rows)
  float* Ps[2];
  float* A;
  float* Db_out;          // X_{k+1}'s split (ld ldd)
  float* Ds_out;
  int64_t ldd;
  int32_t* info;
};

struct StepTile {
  int kind;               // 0: panel P(i); 1: update U(i, j)
  int i, j;
};

// The tiles of CTAs 1 .. g (g = gridDim.x - 1): the panel tiles P(k+1) .. P(T-1) dealt round
// robin (P(k+1+q) to CTA 1 + q % g; CTA 0 computes P(k+1) too, but only for its own use), then the
// updates of the trailing m x m block (m = T - k - 1) without (k+1, k+1), taken column by column,
// each column top to bottom, and cut into g contiguous ranges. Every CTA does its panel tiles
// first.
struct TileList {
  int n_p;                // this CTA's panel tiles
  int u_first;            // its first update tile (index into the update order)
  int n_tiles;
};

__device__ __forceinline__ TileList tile_list(const StepParams& p) {
  if (blockIdx.x == 0) return {1, 0, 2};
  const int m = p.T - p.k - 1;
  const int g = static_cast<int>(gridDim.x) - 1, c = static_cast<int>(blockIdx.x) - 1;
  const int n_u = m * (m + 1) / 2 - 1;
  const int n_p = c < m ? (m - c + g - 1) / g : 0;
  const int u_first = static_cast<int>(static_cast<int64_t>(c) * n_u / g);
  const int u_end = static_cast<int>(static_cast<int64_t>(c + 1) * n_u / g);
  return {n_p, u_first, n_p + u_end - u_first};
}

// update tile u of the order above
__device__ __forceinline__ StepTile update_tile(const StepParams& p, int u) {
  const int m = p.T - p.k - 1;
  const int v = u + 1;                                          // (k+1, k+1) is index 0
  auto off = [m](int c) { return c * m - c * (c - 1) / 2; };   // first index of column c
  const double b = 2.0 * m + 1.0;
  int c = static_cast<int>((b - sqrt(fmax(b * b - 8.0 * v, 0.0))) * 0.5);
  c = c < 0 ? 0 : (c > m - 1 ? m - 1 : c);
  while (c > 0 && off(c) > v) --c;
  while (c < m - 1 && off(c + 1) <= v) ++c;
  return {1, p.k + 1 + c + (v - off(c)), p.k + 1 + c};
}

__device__ __forceinline__ StepTile step_tile(const StepParams& p, const TileList& tl, int t) {
  if (blockIdx.x == 0) return t == 0 ? StepTile{0, p.k + 1, p.k} : StepTile{1, p.k + 1, p.k + 1};
  const int g = static_cast<int>(gridDim.x) - 1, c = static_cast<int>(blockIdx.x) - 1;
  if (t < tl.n_p) return {0, p.k + 1 + c + t * g, p.k};
  return update_tile(p, tl.u_first + t - tl.n_p);
}

__device__ __forceinline__ int tile_boxes(const StepParams& p, const StepTile& s) {
  if (s.kind == 0) return 4;
  const int ncol = min(ps::BN, p.n - s.j * ps::BN);
  return min(4, (ncol + 31) / 32);
}
__device__ __forceinline__ bool tile_loads_c(const StepTile& s) { return s.kind == 1; }
// Update tiles write A_ij back, except the next diagonal block (CTA 0 keeps it on chip) and the
// next panel (its split is what the next step reads; with store_l its L overwrites it anyway).
__device__ __forceinline__ bool tile_stores_c(const StepParams& p, const StepTile& s) {
  if (s.kind == 0) return p.store_l != 0;
  return s.j != p.k + 1;
}

// CTA 0's update of the next diagonal block, boxes j0 .. j1-1 (32 columns each), by one warpgroup
// (TMEM lane = row r): Ld = C - acc on the lower part, identity outside the block's nbd x nbd, in
// the diagonal block's shared layout. Each finished box is handed back to the C-box thread. A lost
// wait stops the whole warpgroup (named barrier bar_id over its 128 threads).
__device__ __forceinline__ void diag_update_boxes(int j0, int j1, uint32_t t_acc, const uint8_t* cs,
                                                  float* Ld, int r, int nbx, int nbd,
                                                  uint64_t* cbox, uint64_t* ready, uint32_t& tok_ph,
                                                  volatile int* abort_flag, int32_t* info,
                                                  uint32_t bar_id) {
  const uint32_t rsw = static_cast<uint32_t>(r & 7);
  bool stop = false;
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    uint32_t vm[32], vc[32];
    tmem_ld_32x32b_x32(t_acc + j * 32, vm);
    tmem_ld_32x32b_x32(t_acc + 128 + j * 32, vc);
    tmem_wait_ld();
    const bool have = j < nbx;
    const bool okc =
        !have || (!stop && mbar_wait_bounded(&cbox[j], (tok_ph >> j) & 1u, abort_flag, info));
    if (have && okc) tok_ph ^= 1u << j;
    const uint8_t* rowp = cs + j * ps::kBoxBytes + r * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (have && okc)
        o = *reinterpret_cast<const float4*>(rowp + ((static_cast<uint32_t>(u) ^ rsw) << 4));
      const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 32 * j + 4 * u + e;
        const float v = ov[e] - (__uint_as_float(vm[4 * u + e]) + __uint_as_float(vc[4 * u + e]));
        Ld[r * la::kLd + c] = (r < nbd && c < nbd) ? (c <= r ? v : 0.f) : (r == c ? 1.f : 0.f);
      }
    }
    stop = named_barrier_or(bar_id, 128, !okc || *abort_flag);
    if (have && !stop) mbar_arrive(&ready[j]);
  }
}

__global__ void __launch_bounds__(ps::kThreads, 1)
potrf_step_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tLb,
                  const __grid_constant__ CUtensorMap tLs, const __grid_constant__ CUtensorMap tP0b,
                  const __grid_constant__ CUtensorMap tP0s, const __grid_constant__ CUtensorMap tP1b,
                  const __grid_constant__ CUtensorMap tP1s, const __grid_constant__ CUtensorMap tDb,
                  const __grid_constant__ CUtensorMap tDs, StepParams p) {
  using namespace ps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ __align__(8) uint64_t cbox[4];        // box j may be written (and holds C if loaded)
  __shared__ __align__(8) uint64_t ready[4];       // box j written by the epilogue
  __shared__ __align__(8) uint64_t opnd_ready;     // CTA 0: L_{k+1,k}'s split is in shared memory
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ float4 stepA[256];                    // diagonal block: per factor step, L entries
  __shared__ float4 stepX[256];                    // diagonal block: per factor step, X entries
  __shared__ int bad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TileList tl = tile_list(p);
  const int n_tiles = tl.n_tiles;
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
    mbar_init(&opnd_ready, 128);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32 * kIssuerWarp) {
    prefetch_tmap(&tA); prefetch_tmap(&tLb); prefetch_tmap(&tLs);
    prefetch_tmap((p.k & 1) ? &tP1b : &tP0b); prefetch_tmap((p.k & 1) ? &tP1s : &tP0s);
    prefetch_tmap(&tDb); prefetch_tmap(&tDs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  griddep_wait();                       // the previous step's results are visible from here
  griddep_launch_dependents();
  // a wait of an earlier step expired: its results are incomplete, do nothing more
  if (threadIdx.x == 0 && p.info != nullptr && *p.info == GPTQ_INFO_TIMEOUT) abort_flag = 1;
  __syncthreads();

  const int k0 = p.k * BN;
  if (warp == 0) {
    // ---------------- A/B producer ----------------
    if (lane == 0) {
      const CUtensorMap* tPb = (p.k & 1) ? &tP1b : &tP0b;
      const CUtensorMap* tPs = (p.k & 1) ? &tP1s : &tP0s;
      int s = 0, issued = 0;
      uint32_t ph = 0;
      for (int t = 0; t < n_tiles && !abort_flag; ++t) {
        if (blockIdx.x == 0 && t == 1) break;      // its operands come from the epilogue
        const StepTile st = step_tile(p, tl, t);
        if (st.kind == 1) {
          if (!flag_wait_bounded(p.flags + st.i, p.k + 1, &abort_flag, p.info) ||
              !flag_wait_bounded(p.flags + st.j, p.k + 1, &abort_flag, p.info))
            break;
          fence_proxy_async_global();
        }
        for (int kb = 0; kb < NK; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, p.info)) goto producer_done;
          uint8_t* sb = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
          if (st.kind == 0) {
            tma_load_2d(sb, tPb, &full_bar[s], kb * BK, st.i * BM);
            tma_load_2d(sb + kPartBytes, tPs, &full_bar[s], kb * BK, st.i * BM);
            tma_load_2d(sb + 2 * kPartBytes, &tDb, &full_bar[s], p.dx + kb * BK, p.dy);
            tma_load_2d(sb + 3 * kPartBytes, &tDs, &full_bar[s], p.dx + kb * BK, p.dy);
          } else {
            tma_load_2d(sb, &tLb, &full_bar[s], k0 + kb * BK, st.i * BM);
            tma_load_2d(sb + kPartBytes, &tLs, &full_bar[s], k0 + kb * BK, st.i * BM);
            tma_load_2d(sb + 2 * kPartBytes, &tLb, &full_bar[s], k0 + kb * BK, st.j * BM);
            tma_load_2d(sb + 3 * kPartBytes, &tLs, &full_bar[s], k0 + kb * BK, st.j * BM);
          }
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    producer_done:
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = make_idesc(/*tf32*/ 2, 0, 0, BM, BN);
      int s = 0;
      uint32_t ph = 0;
      for (int t = 0; t < n_tiles && !abort_flag; ++t) {
        const int buf = t & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ((t >> 1) & 1) ^ 1u, &abort_flag, p.info))
          goto mma_finish;
        tc_fence_after();
        const uint32_t t_main = tmem + buf * 256, t_corr = t_main + 128;
        if (blockIdx.x == 0 && t == 1) {
          // U(k+1, k+1) = A - L L^T with L = L_{k+1,k}: both operands are the split that the panel
          // tile's epilogue left in the idle stage buffers, k-block j at j * 32 KB (big, small)
          if (!mbar_wait_bounded(&opnd_ready, 0, &abort_flag, p.info)) goto mma_finish;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < NK; ++j) {
            const uint32_t base = smem_u32(smem + j * 2 * kPartBytes);
#pragma unroll
            for (int kk = 0; kk < BK / 8; ++kk) {
              const uint64_t lb = smem_desc(base + kk * 32, 16, 1024, kSwizzle128B);
              const uint64_t ls = smem_desc(base + kPartBytes + kk * 32, 16, 1024, kSwizzle128B);
              const uint32_t accum = (j > 0 || kk > 0) ? 1u : 0u;
              tc_mma_tf32(t_corr, lb, ls, idesc, accum);
              tc_mma_tf32(t_corr, ls, lb, idesc, 1u);
              tc_mma_tf32(t_main, lb, lb, idesc, accum);
            }
          }
          tc_commit(&acc_full[buf]);
          continue;
        }
        for (int kb = 0; kb < NK; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, p.info)) goto mma_finish;
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            // K-major, 128-byte swizzle: a K step of 8 tf32 is +32 B inside the 128-byte row
            const uint64_t ab = smem_desc(base + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t as = smem_desc(base + kPartBytes + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bb = smem_desc(base + 2 * kPartBytes + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bs = smem_desc(base + 3 * kPartBytes + kk * 32, 16, 1024, kSwizzle128B);
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
    mma_finish:
      tc_commit(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else if (warp == kIssuerWarp) {
    // ---------------- C boxes: TMA loads for the next tile, stores of finished boxes ----------
    if (lane == 0) {
      uint8_t* cs = smem + kBoxOffset;
      uint32_t rdy_ph = 0;      // per-box parity of the next ready[] completion
      uint32_t rel = 0;         // boxes released at least once
      uint32_t last_ph = 0;     // per-box parity of the latest release's cbox completion
      uint32_t loaded = 0;      // boxes whose latest release loaded C
      auto release = [&](const StepTile& nt, int j) {
        if (rel & (1u << j)) last_ph ^= 1u << j;
        rel |= 1u << j;
        if (tile_loads_c(nt)) {
          loaded |= 1u << j;
          mbar_arrive_expect_tx(&cbox[j], kBoxBytes);
          tma_load_2d(cs + j * kBoxBytes, &tA, &cbox[j], nt.j * BN + 32 * j, nt.i * BM);
        } else {
          loaded &= ~(1u << j);
          mbar_arrive(&cbox[j]);
        }
      };
      const int t_box0 = blockIdx.x == 0 ? 1 : 0;   // CTA 0's panel tile uses no boxes
      if (t_box0 < n_tiles) {
        const StepTile t0 = step_tile(p, tl, t_box0);
        const int nb0 = tile_boxes(p, t0);
        for (int j = 0; j < nb0; ++j) release(t0, j);
      }
      for (int t = t_box0; t < n_tiles; ++t) {
        const StepTile st = step_tile(p, tl, t);
        const int nbx = tile_boxes(p, st);
        const bool store = tile_stores_c(p, st);
        const int col0 = st.kind == 0 ? k0 : st.j * BN;
        StepTile nt{0, 0, 0};
        int nnb = 0;                                 // boxes of the next tile (0: none)
        if (t + 1 < n_tiles) {
          nt = step_tile(p, tl, t + 1);
          nnb = tile_boxes(p, nt);
        }
        bool ok = true;
        for (int j = 0; j < nbx; ++j) {
          if (!mbar_wait_bounded(&ready[j], (rdy_ph >> j) & 1u, &abort_flag, p.info)) {
            ok = false;
            break;
          }
          rdy_ph ^= 1u << j;
          if (store) {
            tma_store_2d(&tA, cs + j * kBoxBytes, col0 + 32 * j, st.i * BM);
            tma_store_commit();
          }
          if (j >= 1) {
            if (store) tma_store_wait_read<1>();     // box j-1 has left shared memory
            if (j - 1 < nnb) release(nt, j - 1);
          }
        }
        if (!ok) break;
        if (store) tma_store_wait_read<0>();
        for (int j = nbx - 1; j < nnb; ++j) release(nt, j);
      }
      tma_store_wait_all();
      for (int j = 0; j < 4; ++j)
        if ((rel & loaded) & (1u << j)) mbar_drain_bounded(&cbox[j], (last_ph >> j) & 1u);
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------- epilogue: TMEM -> C boxes, the tf32 splits, the panel flags ----------
    const int q = warp & 3;
    const int r = q * 32 + lane;                    // row within the tile (= TMEM lane)
    const int et = threadIdx.x - 32 * kEpiWarp0;    // 0..127
    const uint32_t rsw = static_cast<uint32_t>(r & 7);
    uint8_t* cs = smem + kBoxOffset;
    uint32_t tok_ph = 0;                            // per-box parity of the next cbox completion
    for (int t = 0; t < n_tiles; ++t) {
      const StepTile st = step_tile(p, tl, t);
      const int nbx = tile_boxes(p, st);
      const int buf = t & 1;
      const bool ok = mbar_wait_bounded(&acc_full[buf], (t >> 1) & 1, &abort_flag, p.info);
      if (named_barrier_or(kEpiBar, 128, !ok || abort_flag)) break;
      tc_fence_after();
      if (blockIdx.x == 0) {
        const uint32_t t_acc = tmem + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
        if (t == 0) {
          // ---- CTA 0, P(k+1): the split of L_{k+1,k} straight into the stage buffers, as the
          // operands of U(k+1, k+1). (CTA 1 computes the same tile for global memory and the
          // flag, so nothing here has to wait for a store.) ----
#pragma unroll 1
          for (int j = 0; j < 4; ++j) {
            uint32_t vm[32], vc[32];
            tmem_ld_32x32b_x32(t_acc + j * 32, vm);
            tmem_ld_32x32b_x32(t_acc + 128 + j * 32, vc);
            tmem_wait_ld();
            uint8_t* rowp = smem + j * 2 * kPartBytes + r * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              float x[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                x[e] = __uint_as_float(vm[4 * u + e]) + __uint_as_float(vc[4 * u + e]);
              const float4 bg = make_float4(tf32_rna(x[0]), tf32_rna(x[1]), tf32_rna(x[2]),
                                            tf32_rna(x[3]));
              const uint32_t o = (static_cast<uint32_t>(u) ^ rsw) << 4;
              *reinterpret_cast<float4*>(rowp + o) = bg;
              *reinterpret_cast<float4*>(rowp + kPartBytes + o) =
                  make_float4(x[0] - bg.x, x[1] - bg.y, x[2] - bg.z, x[3] - bg.w);
            }
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
          fence_proxy_async_smem();
          mbar_arrive(&opnd_ready);
          continue;
        }
        // ---- CTA 0, U(k+1, k+1): A - L L^T straight into the diagonal block's shared layout
        // (lower part, identity outside the block; it overlaps the stage buffers, idle now that
        // the MMAs are done), boxes 0-1 here and 2-3 by warps 8-11 ----
        diag_update_boxes(0, 2, t_acc, cs, reinterpret_cast<float*>(smem), r, nbx,
                          min(BM, p.n - (p.k + 1) * BM), cbox, ready, tok_ph, &abort_flag, p.info,
                          kEpiBar);
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
        break;
      }
      // where this tile's split goes: L's split (panel tiles) or the next step's panel split
      // (update tiles of block column k+1 below the diagonal); none otherwise
      float* sb = nullptr;
      float* ss = nullptr;
      int64_t sld = 0, scol = 0;
      if (st.kind == 0) {
        sb = p.Lb; ss = p.Ls; sld = p.n; scol = k0;
      } else if (st.j == p.k + 1 && st.i > st.j) {
        // (a select, not an index: indexing a parameter array would copy the parameters to the stack)
        const bool odd = ((p.k + 1) & 1) != 0;
        sb = odd ? p.Pb[1] : p.Pb[0];
        ss = odd ? p.Ps[1] : p.Ps[0];
        sld = BN;
        scol = 0;
      }
      const uint32_t t_main = tmem + buf * 256 + (static_cast<uint32_t>(q * 32) << 16);
      bool stop = false;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        if (j >= nbx) {
          continue;
        }
        uint32_t vm[32], vc[32];
        tmem_ld_32x32b_x32(t_main + j * 32, vm);
        tmem_ld_32x32b_x32(t_main + 128 + j * 32, vc);
        tmem_wait_ld();
        const bool okc = !stop && mbar_wait_bounded(&cbox[j], (tok_ph >> j) & 1u, &abort_flag,
                                                    p.info);
        uint8_t* box = cs + j * kBoxBytes;
        if (okc) {
          tok_ph ^= 1u << j;
          uint8_t* rowp = box + r * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float4* a = reinterpret_cast<float4*>(rowp + ((static_cast<uint32_t>(u) ^ rsw) << 4));
            float x[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              x[e] = __uint_as_float(vm[4 * u + e]) + __uint_as_float(vc[4 * u + e]);
            float4 v;
            if (st.kind == 1) {
              const float4 o = *a;
              v = make_float4(o.x - x[0], o.y - x[1], o.z - x[2], o.w - x[3]);
            } else {
              v = make_float4(x[0], x[1], x[2], x[3]);
            }
            *a = v;
          }
        }
        // every epilogue thread takes the same branch from here (a lost wait stops all of them)
        stop = named_barrier_or(kEpiBar, 128, !okc || abort_flag);
        if (!stop && sb != nullptr) {
          // the tf32 split of the box, written row-contiguous from shared memory
#pragma unroll 4
          for (int s2 = 0; s2 < 8; ++s2) {
            const int f = et + 128 * s2;
            const int br = f >> 3, u = f & 7;
            const int row = st.i * BM + br;
            if (row < p.n) {
              const float4 v = *reinterpret_cast<const float4*>(
                  box + br * 128 + ((static_cast<uint32_t>(u) ^ static_cast<uint32_t>(br & 7)) << 4));
              const float4 bg = make_float4(tf32_rna(v.x), tf32_rna(v.y), tf32_rna(v.z),
                                            tf32_rna(v.w));
              const int64_t off = static_cast<int64_t>(row) * sld + scol + 32 * j + 4 * u;
              *reinterpret_cast<float4*>(sb + off) = bg;
              *reinterpret_cast<float4*>(ss + off) =
                  make_float4(v.x - bg.x, v.y - bg.y, v.z - bg.z, v.w - bg.w);
            }
          }
        }
        if (!stop) {
          fence_proxy_async_smem();
          mbar_arrive(&ready[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      if (stop) break;
      if (st.kind == 0) {
        // publish the panel tile: its split is written (and ordered before the flag)
        fence_proxy_async_global();
        named_barrier_or(kEpiBar, 128, false);
        if (et == 0) {
          __threadfence();
          st_release_gpu(p.flags + st.i, p.k + 1);
        }
      }
    }
  } else if (blockIdx.x == 0 && warp >= kEpiWarp0 + 4 && warp < kEpiWarp0 + 8 && n_tiles == 2) {
    // ---------------- CTA 0: boxes 2-3 of the next diagonal block's update ----------------
    const int r = (warp & 3) * 32 + lane;
    const StepTile st = step_tile(p, tl, 1);
    uint32_t tok_ph = 0;
    const bool ok = mbar_wait_bounded(&acc_full[1], 0, &abort_flag, p.info);
    if (!named_barrier_or(kEpiBar2, 128, !ok || abort_flag)) {   // the same answer for all
      tc_fence_after();
      diag_update_boxes(2, 4, tmem + 256 + (static_cast<uint32_t>((warp & 3) * 32) << 16),
                        smem + kBoxOffset, reinterpret_cast<float*>(smem), r, tile_boxes(p, st),
                        min(BM, p.n - (p.k + 1) * BM), cbox, ready, tok_ph, &abort_flag, p.info,
                        kEpiBar2);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (blockIdx.x != 0 || abort_flag) return;

  // ---------------- CTA 0: factor the diagonal block k+1 (its update left it in L) ----------
  const int kd = (p.k + 1) * BM;
  const int nb = min(BM, p.n - kd);
  float* L = reinterpret_cast<float*>(smem);
  diag_factor_block(L, stepA, stepX, &bad, p.A, p.n, kd, nb, p.Db_out, p.Ds_out, p.ldd, p.info,
                    p.info_base, p.rev_n, p.store_l);
}

gptq_status launch_potrf_fused(float* A, int64_t n, float* Lb, float* Ls, float* Vb, float* Vs,
                               int64_t ld_dinv, bool per_block, float* Pb, float* Ps,
                               int32_t* flags, int32_t* info, int info_base, int rev_n,
                               bool store_l, cudaStream_t stream) {
  using namespace ps;
  const int T = static_cast<int>((n + BM - 1) / BM);
  // the two panel-split parities sit one after the other: rows [0, n) and [n, 2n)
  float* P1b = Pb + n * BN;
  float* P1s = Ps + n * BN;
  CUtensorMap tA, tLb, tLs, tP0b, tP0s, tP1b, tP1s, tDb, tDs;
  gptq_status st;
  auto kmap = [&](CUtensorMap* m, const float* base, int64_t k_ext, int64_t mn_ext, int64_t ld) {
    return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, 4, k_ext, mn_ext, ld, 32, BM,
                          CU_TENSOR_MAP_SWIZZLE_128B);
  };
  if ((st = kmap(&tA, A, n, n, n)) != GPTQ_OK) return st;
  if ((st = kmap(&tLb, Lb, n, n, n)) != GPTQ_OK) return st;
  if ((st = kmap(&tLs, Ls, n, n, n)) != GPTQ_OK) return st;
  if ((st = kmap(&tP0b, Pb, BN, n, BN)) != GPTQ_OK) return st;
  if ((st = kmap(&tP0s, Ps, BN, n, BN)) != GPTQ_OK) return st;
  if ((st = kmap(&tP1b, P1b, BN, n, BN)) != GPTQ_OK) return st;
  if ((st = kmap(&tP1s, P1s, BN, n, BN)) != GPTQ_OK) return st;
  if (per_block) {
    if ((st = kmap(&tDb, Vb, n, n, ld_dinv)) != GPTQ_OK) return st;
    if ((st = kmap(&tDs, Vs, n, n, ld_dinv)) != GPTQ_OK) return st;
  } else {
    // two 128 x 128 scratch blocks, one per parity of the step, stacked
    if ((st = kmap(&tDb, Vb, BN, 2 * BM, ld_dinv)) != GPTQ_OK) return st;
    if ((st = kmap(&tDs, Vs, BN, 2 * BM, ld_dinv)) != GPTQ_OK) return st;
  }
  if ((st = set_max_dynamic_smem(reinterpret_cast<const void*>(potrf_step_kernel), kSmemBytes)) !=
      GPTQ_OK)
    return st;
  const int sms = num_sms();
  for (int k = 0; k + 1 < T; ++k) {
    StepParams p;
    p.n = static_cast<int>(n);
    p.T = T;
    p.k = k;
    p.store_l = store_l ? 1 : 0;
    p.rev_n = rev_n;
    p.info_base = info_base;
    const int m = T - k - 1;
    const int n_u = m * (m + 1) / 2 - 1;              // update tiles for CTAs 1 ..
    // CTAs 1 .. g, each with at least one tile: the panel tiles alone when they outnumber the
    // updates (the last steps), else every CTA takes at least one update
    const int g_want = m > n_u ? m : n_u;
    if (per_block) {
      p.dx = k * BN;
      p.dy = k * BM;
      const int64_t off = static_cast<int64_t>(k + 1) * BM * ld_dinv + (k + 1) * BN;
      p.Db_out = Vb + off;
      p.Ds_out = Vs + off;
    } else {
      p.dx = 0;
      p.dy = (k & 1) * BM;
      const int64_t off = static_cast<int64_t>((k + 1) & 1) * BM * ld_dinv;
      p.Db_out = Vb + off;
      p.Ds_out = Vs + off;
    }
    p.ldd = ld_dinv;
    p.flags = flags;
    p.Lb = Lb;
    p.Ls = Ls;
    p.Pb[0] = Pb; p.Pb[1] = P1b;
    p.Ps[0] = Ps; p.Ps[1] = P1s;
    p.A = A;
    p.info = info;
    const int grid = 1 + (g_want < sms - 1 ? g_want : sms - 1);
    if ((st = launch_pdl(potrf_step_kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, tA, tLb,
                         tLs, tP0b, tP0s, tP1b, tP1s, tDb, tDs, p)) != GPTQ_OK)
      return st;
  }
  return GPTQ_OK;
}

}  // namespace gptq
