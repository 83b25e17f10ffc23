// S1 -- proxy Hessian accumulation S += X^T X (lower triangle), X token-major [n_tokens x ldx].
//
// "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)", section "Goal": the input covariance
// is the proxy Hessian; "Part 3: Adaptive Rounding: GPTQ", "Algorithm GPTQ": H = X X^T + lambda I.
//
// bf16 path: a persistent tcgen05 SYRK on CTA pairs (the 2-SM form, cta_group::2). The output is
// cut into 256 x 256 lower-triangle super-tiles; each pair of CTAs (a cluster of 2 on two SMs) owns
// one super-tile per round and walks the whole token range for it, so all pairs read the same token
// slab at about the same time (fetched from HBM once, served to the others from L2). Per 128-token
// stage each CTA brings, by TMA with 128-byte swizzle, the 128 channels of its half of the rows (A)
// and of its half of the columns (B) into its own shared memory (64 KB, three stages); both
// operands are MN-major (channels contiguous), which tcgen05 reads directly, and on a diagonal
// super-tile A doubles as B. The first CTA of the pair issues eight 256 x 256 x 16 MMAs per stage;
// each CTA's TMEM receives its 128 rows. Per SM this moves half the operand bytes of a 128 x 256
// single-SM tile. Long stages matter: with 32-token stages (4 KB boxes) the same pipeline kept the
// tensor cores waiting for operands a third of the time.
//
// The tensor core adds each MMA's products into its fp32 accumulator with a rounding biased
// toward zero, so the relative error of one TMEM sum grows with the number of MMAs folded into it
// (about 6e-8 per MMA measured on B200). Every kChunkStages stages (2048 tokens) the chunk sum is
// handed to eight epilogue warps in each CTA, which add it into fp32 registers with IEEE adds while
// the MMAs fill the other of two chunk buffers (2 x 256 TMEM columns); at the end of the super-tile
// the registers are added into S once. Each super-tile belongs to one pair: deterministic.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace syrk {
constexpr int kBK = 128;                   // tokens per stage
constexpr int kStages = 3;
constexpr int kBoxCh = 64;                 // channels per TMA box (128 bytes of bf16)
constexpr int kBoxBytes = kBoxCh * kBK * 2;          // 16 KB
constexpr int kHalfBytes = 2 * kBoxBytes;            // 128 channels
constexpr int kStageBytes = 2 * kHalfBytes;          // A half + B half: 64 KB per CTA
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kThreads = 320;              // warp 0 TMA, warp 1 MMA (first CTA), warps 2-9 fold
constexpr uint32_t kTmemCols = 512;        // two 256-column chunk accumulators (128 rows each)
constexpr int kChunkStages = 2048 / kBK;   // 2048 tokens per TMEM chunk sum
constexpr uint32_t kIdesc = make_idesc(/*bf16*/ 1, /*A MN-major*/ 1, /*B MN-major*/ 1, 256, 256);
constexpr int kEpiWarps = 8;
}  // namespace syrk

__device__ __forceinline__ void decode_lower(int st, int& I, int& J) {
  int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(st) + 1.0f) - 1.0f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= st) ++i;
  while (i * (i + 1) / 2 > st) --i;
  I = i;
  J = st - i * (i + 1) / 2;
}

// The order in which the pairs take super-tiles. The pairs of one round (consecutive super-tiles)
// stream the same token slab at about the same time, so what HBM delivers per round is the
// channel blocks their super-tiles touch. Row-major order over the lower triangle gives a round
// one block row and ~n_pairs block columns (~75 distinct blocks at 49152 channels); here the
// triangle is cut into panels of kPanel block rows, taken block column by block column, so a round
// spans about kPanel rows and n_pairs / kPanel columns (~18 distinct blocks).
constexpr int kPanel = 8;
__device__ __forceinline__ void decode_panel(int st, int T, int& I, int& J) {
  int p = 0;
  while ((p + 1) * kPanel < T && ((p + 1) * kPanel) * ((p + 1) * kPanel + 1) / 2 <= st) ++p;
  const int r0 = p * kPanel, h = min(kPanel, T - r0);
  int idx = st - r0 * (r0 + 1) / 2;
  if (idx < r0 * h) {                       // block columns left of the panel: full height
    I = r0 + idx % h;
    J = idx / h;
    return;
  }
  idx -= r0 * h;                            // the panel's own triangle, column by column
  int q = 0;
  while (idx >= h - q) {
    idx -= h - q;
    ++q;
  }
  I = r0 + q + idx;
  J = r0 + q;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(syrk::kThreads, 1)
hessian_syrk_bf16_tc(const __grid_constant__ CUtensorMap tmap, float* __restrict__ S, int cols,
                     int n_kblocks, int n_super, int n_s, int32_t* info) {
  using namespace syrk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);

  __shared__ __align__(8) uint64_t full_bar[kStages];    // used in the first CTA
  __shared__ __align__(8) uint64_t empty_bar[kStages];   // in both CTAs
  __shared__ __align__(8) uint64_t acc_full[2];          // in both CTAs
  __shared__ __align__(8) uint64_t acc_empty[2];         // used in the first CTA
  __shared__ __align__(8) uint64_t mma_done;             // used in the first CTA
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmap);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base_sh, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      for (int st = pair; st < n_super && !abort_flag; st += n_pairs) {
        int I, J;
        decode_panel(st, n_s, I, J);
        const bool diag = (I == J);
        const uint32_t bytes = diag ? kHalfBytes : kStageBytes;   // this CTA's share
        for (int kb = 0; kb < n_kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag, info)) goto producer_done;
          uint8_t* a = smem + s * kStageBytes;
          uint8_t* b = a + kHalfBytes;
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * bytes);
#pragma unroll
          for (int q = 0; q < 2; ++q)
            tma_load_2d_pair(a + q * kBoxBytes, &tmap, fb,
                             I * 256 + static_cast<int>(rank) * 128 + q * kBoxCh, kb * kBK);
          if (!diag) {
#pragma unroll
            for (int q = 0; q < 2; ++q)
              tma_load_2d_pair(b + q * kBoxBytes, &tmap, fb,
                               J * 256 + static_cast<int>(rank) * 128 + q * kBoxCh, kb * kBK);
          }
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    producer_done:
      // the first CTA's full barriers count both CTAs' copies: let every issued copy land
      if (leader) {
        for (long long i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
          mbar_drain_bounded(&full_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (first CTA of the pair) ----------------
      int s = 0;
      uint32_t ph = 0;
      int chunk = 0;
      for (int st = pair; st < n_super && !abort_flag; st += n_pairs) {
        int I, J;
        decode_panel(st, n_s, I, J);
        const bool diag = (I == J);
        for (int kc = 0; kc < n_kblocks; kc += kChunkStages, ++chunk) {
          const int buf = chunk & 1;
          if (!mbar_wait_bounded(&acc_empty[buf], ((chunk >> 1) & 1) ^ 1u, &abort_flag, info))
            goto mma_done_label;
          tc_fence_after();
          const int kc_end = min(n_kblocks, kc + kChunkStages);
          for (int kb = kc; kb < kc_end; ++kb) {
            if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, info)) goto mma_done_label;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
            const uint32_t b_addr = diag ? a_addr : a_addr + kHalfBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t adesc = smem_desc(a_addr + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
              const uint64_t bdesc = smem_desc(b_addr + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
              tc_mma_f16_pair(tmem + buf * 256, adesc, bdesc, kIdesc,
                              (kb > kc || kk > 0) ? 1u : 0u);
            }
            tc_commit_pair_mc(&empty_bar[s], 0x3);
            if (++s == kStages) { s = 0; ph ^= 1u; }
          }
          tc_commit_pair_mc(&acc_full[buf], 0x3);
        }
      }
    mma_done_label:
      tc_commit_pair(&mma_done);
      mbar_drain_bounded(&mma_done, 0);
    }
  } else {
    // ---------- fold chunk sums into registers; add the super-tile's rows into S at its end ----
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;     // column half: 0 -> 0..127, 1 -> 128..255
    const uint32_t ae0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    const uint32_t ae1 = mapa_shared(smem_u32(&acc_empty[1]), 0);
    int chunk = 0;
    bool ok = true;
    for (int st = pair; st < n_super && ok && !abort_flag; st += n_pairs) {
      int I, J;
      decode_panel(st, n_s, I, J);
      float acc[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) acc[j] = 0.f;
      for (int kc = 0; kc < n_kblocks; kc += kChunkStages, ++chunk) {
        const int buf = chunk & 1;
        if (!mbar_wait_bounded(&acc_full[buf], (chunk >> 1) & 1, &abort_flag, info)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t0 = tmem + buf * 256 + h * 128 + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t0 + cc * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) acc[cc * 32 + t] += __uint_as_float(v[t]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(buf ? ae1 : ae0);
      }
      if (!ok) break;
      const int i = I * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
      const int j0 = J * 256 + h * 128;
      if (i < cols) {
        float4* row = reinterpret_cast<float4*>(S + static_cast<size_t>(i) * cols + j0);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if (j0 + 4 * t < cols) {
            float4 o = row[t];
            o.x += acc[4 * t + 0];
            o.y += acc[4 * t + 1];
            o.z += acc[4 * t + 2];
            o.w += acc[4 * t + 3];
            row[t] = o;
          }
        }
      }
    }
  }

  // every MMA of the pair has completed (the first CTA waited for them) before either CTA frees
  // its tensor memory or exits
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// fp32 inputs: CUDA-core SYRK on 64 x 64 lower tiles with the token range split over blockIdx.y;
// partial tiles are added into S with atomics (exact fp32 products, fp32 sums).
__global__ void __launch_bounds__(256)
hessian_syrk_f32_simt(const float* __restrict__ X, int64_t ldx, float* __restrict__ S, int cols,
                      int64_t n_tokens, int64_t tok_per_split) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  int I, J;
  decode_lower(blockIdx.x, I, J);
  const int i0 = I * 64, j0 = J * 64;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.y) * tok_per_split;
  const int64_t t_end = min(n_tokens, t_begin + tok_per_split);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int64_t t0 = t_begin; t0 < t_end; t0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e >> 6, c = e & 63;
      const int64_t t = t0 + kk;
      const bool tok_ok = t < t_end;
      As[kk][c] = (tok_ok && i0 + c < cols) ? X[t * ldx + i0 + c] : 0.f;
      Bs[kk][c] = (tok_ok && j0 + c < cols) ? X[t * ldx + j0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty * 4 + u];
        b[u] = Bs[kk][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= cols) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int j = j0 + tx * 4 + v;
      if (j < cols) atomicAdd(S + static_cast<size_t>(i) * cols + j, acc[u][v]);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------------

gptq_status launch_hessian_bf16(float* S, int64_t cols, const void* X, int64_t n_tokens,
                                int64_t ldx, int32_t* info, cudaStream_t stream) {
  using namespace syrk;
  CUtensorMap tmap;
  gptq_status st = encode_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, 2,
                                  static_cast<uint64_t>(cols), static_cast<uint64_t>(n_tokens),
                                  static_cast<uint64_t>(ldx), kBoxCh, kBK,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GPTQ_OK) return st;
  if ((st = set_max_dynamic_smem(reinterpret_cast<const void*>(hessian_syrk_bf16_tc),
                                 kSmemBytes)) != GPTQ_OK)
    return st;
  // lower 256 x 256 super-tiles, one per CTA pair per round
  const int n_s = static_cast<int>((cols + 255) / 256);
  const int n_super = n_s * (n_s + 1) / 2;
  const int64_t n_kb = (n_tokens + kBK - 1) / kBK;
  if (n_kb > INT32_MAX / kBK) return GPTQ_EUNSUPPORTED;
  const int max_pairs = num_sms() / 2;
  const int pairs = n_super < max_pairs ? n_super : max_pairs;
  hessian_syrk_bf16_tc<<<2 * pairs, kThreads, kSmemBytes, stream>>>(
      tmap, S, static_cast<int>(cols), static_cast<int>(n_kb), n_super, n_s, info);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

gptq_status launch_hessian_f32(float* S, int64_t cols, const float* X, int64_t n_tokens,
                               int64_t ldx, cudaStream_t stream) {
  const int n_t = static_cast<int>((cols + 63) / 64);
  const int n_tiles = n_t * (n_t + 1) / 2;
  // enough splits to give every SM a few CTAs, each with at least 256 tokens
  int64_t splits = (4 * num_sms() + n_tiles - 1) / n_tiles;
  const int64_t max_splits = (n_tokens + 255) / 256;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  if (splits > 65535) splits = 65535;
  int64_t per = (n_tokens + splits - 1) / splits;
  per = (per + 15) / 16 * 16;
  splits = (n_tokens + per - 1) / per;
  dim3 grid(n_tiles, static_cast<unsigned>(splits));
  hessian_syrk_f32_simt<<<grid, 256, 0, stream>>>(X, ldx, S, static_cast<int>(cols), n_tokens, per);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ECUDA;
}

}  // namespace gptq
